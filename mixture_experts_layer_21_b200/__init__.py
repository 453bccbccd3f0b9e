"""Python binding of the B200 fused MoE expert layer (``libmoe_b200.so``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. PyTorch provides device memory and streams. The functions carry the C
entry points' names (see ``include/moe.h``); each takes and returns torch
tensors on the current CUDA device and launches on the current stream.

There is no fallback: if the shared library is missing the import fails.
Build it with ``python mixture_experts_layer_21_b200/build.py``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: run `python mixture_experts_layer_21_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

MOE_OK = 0
STATUS = ["MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED", "MOE_ERR_ALIGNMENT",
          "MOE_ERR_WORKSPACE_TOO_SMALL", "MOE_ERR_CUDA", "MOE_ERR_DEVICE", "MOE_ERR_TIMEOUT",
          "MOE_ERR_NOT_PREPARED"]
ACT = {"silu": 0, "situ": 1, "swigluoai": 2}
WFMT = {"bf16": 0, "mxfp4": 1, "nvfp4": 2}

# Every symbol include/moe.h declares.
EXPORTS = ["moe_status_string", "moe_version", "moe_route_topk", "moe_permute_workspace_size",
           "moe_permute", "moe_grouped_gemm_workspace_size", "moe_grouped_gemm", "moe_act_and_mul",
           "moe_combine", "moe_quantize_nvfp4", "moe_prepared_weight_bytes", "moe_prepare_weights",
           "moe_forward_workspace_size", "moe_forward", "moe_get_device_error", "moe_permute_noalloc",
           "moe_permute_noalloc_status", "moe_grouped_gemm_nvfp4", "moe_quantize_mxfp8", "moe_route_topk_grouped",
           "moe_bias_act_and_mul", "moe_forward_workspace_size_args"]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = STATUS[status] if 0 <= status < len(STATUS) else str(status)
        super().__init__(f"{where}: {name}")


class moe_weight_t(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("G", ctypes.c_int32), ("N", ctypes.c_int32),
                ("K", ctypes.c_int32), ("data", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("alpha", ctypes.c_void_p), ("kdata", ctypes.c_void_p), ("kscale", ctypes.c_void_p),
                ("kalpha", ctypes.c_void_p)]


class moe_act_params_t(ctypes.Structure):
    _fields_ = [("act", ctypes.c_int32), ("situ_alpha", ctypes.c_float), ("situ_beta", ctypes.c_float)]


class moe_act_ex_t(ctypes.Structure):
    _fields_ = [("act", ctypes.c_int32), ("situ_alpha", ctypes.c_float), ("situ_beta", ctypes.c_float),
                ("swiglu_alpha", ctypes.c_float), ("swiglu_beta", ctypes.c_float),
                ("swiglu_limit", ctypes.c_float)]


class moe_forward_args_t(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("router_logits", ctypes.c_void_p),
                ("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("B", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("replica_src", ctypes.c_void_p),
                ("w_gate", moe_weight_t), ("w_up", moe_weight_t), ("w_down", moe_weight_t),
                ("act", moe_act_params_t), ("apply_topk_in_fc1", ctypes.c_int32),
                ("act_quant", ctypes.c_int32), ("out", ctypes.c_void_p),
                ("topk_ids_out", ctypes.c_void_p), ("topk_w_out", ctypes.c_void_p),
                ("T_max", ctypes.c_int32), ("stage_events", ctypes.c_void_p),
                ("routing", ctypes.c_int32), ("routing_bias", ctypes.c_void_p),
                ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float),
                ("topk_ids_in", ctypes.c_void_p), ("topk_w_in", ctypes.c_void_p),
                ("apply_router_weight_on_input", ctypes.c_int32),
                ("swiglu_alpha", ctypes.c_float), ("swiglu_beta", ctypes.c_float),
                ("swiglu_limit", ctypes.c_float),
                ("bias_gate", ctypes.c_void_p), ("bias_up", ctypes.c_void_p), ("bias_down", ctypes.c_void_p)]

ROUTING = {"renormalize": 0, "deepseek_v3": 1, "given": 2}

MOE_FWD_STAGE_EVENTS = 7


_P, _I, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_sig = {
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_version": (ctypes.c_char_p, []),
    "moe_route_topk": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "moe_permute_workspace_size": (_S, [_I, _I, _I, _I]),
    "moe_permute": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P, _P, _I, _P, _S, _P]),
    "moe_grouped_gemm_workspace_size": (_S, [_I, ctypes.POINTER(moe_weight_t)]),
    "moe_grouped_gemm": (_I, [_P, _I, ctypes.POINTER(moe_weight_t), _P, _P, _P, _S, _P]),
    "moe_act_and_mul": (_I, [_P, _P, _P, _I, _I, moe_act_params_t, _P, _P]),
    "moe_combine": (_I, [_P, _P, _P, _I, _I, _I, _P, _P]),
    "moe_quantize_nvfp4": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P]),
    "moe_prepared_weight_bytes": (_S, [ctypes.POINTER(moe_weight_t)]),
    "moe_prepare_weights": (_I, [ctypes.POINTER(moe_weight_t), _P, _S, _P]),
    "moe_forward_workspace_size": (_S, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "moe_forward": (_I, [ctypes.POINTER(moe_forward_args_t), _P, _S, _P]),
    "moe_get_device_error": (_I, [_P, _P]),
    "moe_permute_noalloc": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P, _P, _I, _P]),
    "moe_permute_noalloc_status": (_I, [_P]),
    "moe_grouped_gemm_nvfp4": (_I, [_P, _P, _P, _I, ctypes.POINTER(moe_weight_t), _P, _P, _P, _S, _P]),
    "moe_quantize_mxfp8": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "moe_route_topk_grouped": (_I, [_P, _P, _I, _I, _I, _I, _I, ctypes.c_float, _P, _P, _P]),
    "moe_bias_act_and_mul": (_I, [_P, _P, _I, _P, _P, _P, _I, _P, _I, _I, ctypes.POINTER(moe_act_ex_t), _P, _P]),
    "moe_forward_workspace_size_args": (_S, [ctypes.POINTER(moe_forward_args_t)]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


def lib() -> ctypes.CDLL:
    return _lib


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoEError(status, where)


def version() -> str:
    return _lib.moe_version().decode()


def status_string(s: int) -> str:
    return _lib.moe_status_string(s).decode()


# ---------------------------------------------------------------------------- weights

@dataclass
class Weight:
    """One projection's weights on the device plus their prepared kernel-format copy.

    ``data``: bf16 [G,N,K] or uint8 packed e2m1 [G,N,K/2]; ``scale``: uint8 e8m0
    [G,N,K/32] (MXFP4) or e4m3 [G,N,K/16] (NVFP4); ``alpha``: fp32 [G] or None.
    """

    fmt: str
    data: torch.Tensor
    scale: torch.Tensor | None = None
    alpha: torch.Tensor | None = None
    prepared: torch.Tensor | None = None
    desc: moe_weight_t = field(default_factory=moe_weight_t)

    def __post_init__(self):
        d = self.desc
        d.fmt = WFMT[self.fmt]
        d.G, d.N = self.data.shape[0], self.data.shape[1]
        d.K = self.data.shape[2] * (1 if self.fmt == "bf16" else 2)
        d.data, d.scale, d.alpha = _ptr(self.data), _ptr(self.scale), _ptr(self.alpha)

    @property
    def G(self):
        return self.desc.G

    @property
    def N(self):
        return self.desc.N

    @property
    def K(self):
        return self.desc.K

    @classmethod
    def from_host(cls, ws, device="cuda") -> "Weight":
        """From a ``workloads.WeightSet`` (CPU) to the device."""
        mv = lambda t: None if t is None else t.to(device, non_blocking=False).contiguous()
        return cls(ws.fmt, mv(ws.data), mv(ws.scale), mv(ws.alpha))


def moe_prepare_weights(w: Weight, stream=None) -> Weight:
    """S0: kernel-format copy of FP4 weights (no-op for BF16). Synchronises."""
    if w.fmt == "bf16":
        return w
    nbytes = _lib.moe_prepared_weight_bytes(ctypes.byref(w.desc))
    w.prepared = torch.empty(nbytes, dtype=torch.uint8, device=w.data.device)
    _check(_lib.moe_prepare_weights(ctypes.byref(w.desc), _ptr(w.prepared), nbytes, _stream(stream)),
           "moe_prepare_weights")
    return w


# ---------------------------------------------------------------------------- steps

def moe_route_topk(logits: torch.Tensor, topk: int, ids=None, w=None, stream=None):
    T, E = logits.shape
    ids = ids if ids is not None else torch.empty(T, topk, dtype=torch.int32, device=logits.device)
    w = w if w is not None else torch.empty(T, topk, dtype=torch.float32, device=logits.device)
    _check(_lib.moe_route_topk(_ptr(logits), T, E, topk, _ptr(ids), _ptr(w), _stream(stream)),
           "moe_route_topk")
    return ids, w


def moe_route_topk_grouped(logits: torch.Tensor, topk: int, n_group: int, topk_group: int, bias=None,
                           routed_scaling_factor: float = 1.0, ids=None, w=None, stream=None):
    """DeepSeekV3 routing (grouped top-k on sigmoid scores, bias for selection only)."""
    T, E = logits.shape
    ids = ids if ids is not None else torch.empty(T, topk, dtype=torch.int32, device=logits.device)
    w = w if w is not None else torch.empty(T, topk, dtype=torch.float32, device=logits.device)
    _check(_lib.moe_route_topk_grouped(_ptr(logits), _ptr(bias), T, E, topk, n_group, topk_group,
                                       routed_scaling_factor, _ptr(ids), _ptr(w), _stream(stream)),
           "moe_route_topk_grouped")
    return ids, w


def permute_workspace(T: int, topk: int, E: int, B: int, device="cuda") -> torch.Tensor:
    n = _lib.moe_permute_workspace_size(T, topk, E, B)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def moe_permute(topk_ids, topk_w, E: int, B: int = 0, replica_src=None, x=None, M_alloc=None,
                ws=None, stream=None, out=None):
    """``out``: optional dict of caller-allocated outputs (any of cu_seqlens, perm_token,
    perm_w, inv_perm, x_perm [M_alloc,H]); the others are allocated here."""
    T, k = topk_ids.shape
    dev = topk_ids.device
    NvS = T * k
    out = out or {}
    M_alloc = NvS if M_alloc is None else M_alloc
    ws = ws if ws is not None else permute_workspace(T, k, E, B, dev)
    def buf(name, shape, dtype):
        t = out.get(name)
        return t if t is not None else torch.empty(shape, dtype=dtype, device=dev)

    cu = buf("cu_seqlens", (E + B,), torch.int32)
    perm_token = buf("perm_token", (NvS,), torch.int32)
    perm_w = buf("perm_w", (NvS,), torch.float32)
    inv = buf("inv_perm", (T, k), torch.int32)
    x_perm = None
    H = 0
    if x is not None:
        H = x.shape[1]
        x_perm = out.get("x_perm")
        if x_perm is None:
            x_perm = torch.zeros(M_alloc, H, dtype=x.dtype, device=dev)
        M_alloc = x_perm.shape[0]
    _check(_lib.moe_permute(_ptr(topk_ids), _ptr(topk_w), T, k, E, B, _ptr(replica_src), _ptr(x), H,
                            _ptr(cu), _ptr(perm_token), _ptr(perm_w), _ptr(inv), _ptr(x_perm), M_alloc,
                            _ptr(ws), ws.numel(), _stream(stream)), "moe_permute")
    return dict(cu_seqlens=cu, perm_token=perm_token, perm_w=perm_w, inv_perm=inv, x_perm=x_perm, ws=ws)


def moe_grouped_gemm(a: torch.Tensor, w: Weight, cu_seqlens: torch.Tensor, out=None, ws=None,
                     stream=None) -> torch.Tensor:
    M = a.shape[0]
    out = out if out is not None else torch.empty(M, w.N, dtype=torch.bfloat16, device=a.device)
    if ws is None:
        n = _lib.moe_grouped_gemm_workspace_size(M, ctypes.byref(w.desc))
        ws = torch.zeros(n, dtype=torch.uint8, device=a.device)
    _check(_lib.moe_grouped_gemm(_ptr(a), M, ctypes.byref(w.desc), _ptr(cu_seqlens), _ptr(out),
                                 _ptr(ws), ws.numel(), _stream(stream)), "moe_grouped_gemm")
    return out


def moe_grouped_gemm_nvfp4(a_codes: torch.Tensor, a_sb: torch.Tensor, a_s: torch.Tensor, w: Weight,
                           cu_seqlens: torch.Tensor, out=None, ws=None, stream=None) -> torch.Tensor:
    """Block-scaled grouped GEMM on NVFP4 activations (codes [M,K/2], e4m3 scales [M,K/16],
    row scales [M]) and prepared NVFP4 weights; bf16 out [M,N]."""
    M = a_codes.shape[0]
    out = out if out is not None else torch.empty(M, w.N, dtype=torch.bfloat16, device=a_codes.device)
    ws = ws if ws is not None else torch.zeros(256, dtype=torch.uint8, device=a_codes.device)
    _check(_lib.moe_grouped_gemm_nvfp4(_ptr(a_codes), _ptr(a_sb), _ptr(a_s), M, ctypes.byref(w.desc),
                                       _ptr(cu_seqlens), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_grouped_gemm_nvfp4")
    return out


def act_params(act: str = "silu", situ_alpha: float = 1.0, situ_beta: float = 1.0) -> moe_act_params_t:
    return moe_act_params_t(ACT[act], situ_alpha, situ_beta)


def moe_act_and_mul(gate, up, perm_w=None, act: str = "silu", situ_alpha=1.0, situ_beta=1.0, out=None,
                    stream=None):
    M, I = gate.shape
    out = out if out is not None else torch.empty_like(gate)
    _check(_lib.moe_act_and_mul(_ptr(gate), _ptr(up), _ptr(perm_w), M, I,
                                act_params(act, situ_alpha, situ_beta), _ptr(out), _stream(stream)),
           "moe_act_and_mul")
    return out


def act_ex(act: str = "silu", situ_alpha: float = 1.0, situ_beta: float = 1.0, swiglu_alpha: float = 1.702,
           swiglu_beta: float = 1.0, swiglu_limit: float | None = 7.0) -> moe_act_ex_t:
    """Activation and parameters; ``swiglu_limit=None`` means no clamp (+inf)."""
    lim = float("inf") if swiglu_limit is None else swiglu_limit
    return moe_act_ex_t(ACT[act], situ_alpha, situ_beta, swiglu_alpha, swiglu_beta, lim)


def moe_bias_act_and_mul(gate, up, cu_seqlens, bias_gate=None, bias_up=None, perm_w=None, act: str = "silu",
                         situ_alpha=1.0, situ_beta=1.0, swiglu_alpha=1.702, swiglu_beta=1.0, swiglu_limit=7.0,
                         out=None, stream=None):
    """S4 with per-expert biases (fp32 [G,I]) and any activation, SWIGLUOAI included. gate/up
    bf16 or fp32 [M,I]; bf16 out [M,I]; rows past cu_seqlens[-1] come out zero."""
    M, I = gate.shape
    out = out if out is not None else torch.empty(M, I, dtype=torch.bfloat16, device=gate.device)
    a = act_ex(act, situ_alpha, situ_beta, swiglu_alpha, swiglu_beta, swiglu_limit)
    _check(_lib.moe_bias_act_and_mul(_ptr(gate), _ptr(up), 1 if gate.dtype == torch.float32 else 0, _ptr(bias_gate),
                                     _ptr(bias_up), _ptr(cu_seqlens), cu_seqlens.numel(), _ptr(perm_w), M, I,
                                     ctypes.byref(a), _ptr(out), _stream(stream)), "moe_bias_act_and_mul")
    return out


def moe_combine(y_perm, inv_perm, topk_w=None, out=None, stream=None):
    T, k = inv_perm.shape
    H = y_perm.shape[1]
    out = out if out is not None else torch.empty(T, H, dtype=torch.bfloat16, device=y_perm.device)
    _check(_lib.moe_combine(_ptr(y_perm), _ptr(inv_perm), _ptr(topk_w), T, k, H, _ptr(out),
                            _stream(stream)), "moe_combine")
    return out


def moe_quantize_nvfp4(x: torch.Tensor, deq: bool = True, stream=None):
    R, K = x.shape
    dev = x.device
    codes = torch.empty(R, K // 2, dtype=torch.uint8, device=dev)
    sb = torch.empty(R, K // 16, dtype=torch.uint8, device=dev)
    s = torch.empty(R, dtype=torch.float32, device=dev)
    d = torch.empty(R, K, dtype=torch.float16, device=dev) if deq else None
    _check(_lib.moe_quantize_nvfp4(_ptr(x), 1 if x.dtype == torch.float32 else 0, R, K, _ptr(codes),
                                   _ptr(sb), _ptr(s), _ptr(d), _stream(stream)), "moe_quantize_nvfp4")
    return codes, sb, s, d


def moe_quantize_mxfp8(x: torch.Tensor, stream=None):
    """Dynamic MXFP8 quantisation of rows (bf16 or fp32 [R,K]): e4m3 codes [R,K] and e8m0
    scales [R,K/32]."""
    R, K = x.shape
    codes = torch.empty(R, K, dtype=torch.uint8, device=x.device)
    scales = torch.empty(R, K // 32, dtype=torch.uint8, device=x.device)
    _check(_lib.moe_quantize_mxfp8(_ptr(x), 1 if x.dtype == torch.float32 else 0, R, K, _ptr(codes), _ptr(scales),
                                   _stream(stream)), "moe_quantize_mxfp8")
    return codes, scales


def forward_workspace(T_max, H, I, E, B, topk, wfmt="bf16", act_quant=0, device="cuda") -> torch.Tensor:
    n = _lib.moe_forward_workspace_size(T_max, H, I, E, B, topk, WFMT[wfmt], act_quant)
    return torch.zeros(n, dtype=torch.uint8, device=device)


class MoEForward:
    """The fused layer with its weights and a pre-sized workspace (no per-call allocation
    besides the output, which the caller may also pass)."""

    def __init__(self, w_gate: Weight, w_up: Weight, w_down: Weight, E: int, topk: int, B: int = 0,
                 replica_src=None, act: str = "silu", situ_alpha=1.0, situ_beta=1.0,
                 act_quant: int = 0, apply_topk_in_fc1: bool = True, T_max: int = 1,
                 routing: str = "renormalize", routing_bias=None, n_group: int = 1, topk_group: int = 1,
                 routed_scaling_factor: float = 1.0, apply_router_weight_on_input: bool = False,
                 swiglu_alpha: float = 1.702, swiglu_beta: float = 1.0, swiglu_limit: float | None = 7.0,
                 biases=None):
        """``biases``: None, or (bias_gate [E+B,I], bias_up [E+B,I], bias_down [E+B,H]) fp32
        device tensors, each of which may be None; the GEMMs' epilogues apply them."""
        for w in (w_gate, w_up, w_down):
            if w.fmt != "bf16" and w.prepared is None:
                moe_prepare_weights(w)
        self.w_gate, self.w_up, self.w_down = w_gate, w_up, w_down
        self.E, self.topk, self.B = E, topk, B
        self.H, self.I = w_gate.K, w_gate.N
        self.replica_src = replica_src
        self.act = act_params(act, situ_alpha, situ_beta)
        self.act_quant = act_quant
        self.apply_topk_in_fc1 = apply_topk_in_fc1
        self.T_max = T_max
        self.args = moe_forward_args_t()
        a = self.args
        a.swiglu_alpha, a.swiglu_beta = swiglu_alpha, swiglu_beta
        a.swiglu_limit = float("inf") if swiglu_limit is None else swiglu_limit
        self.biases = tuple(biases) if biases is not None else (None, None, None)
        a.bias_gate, a.bias_up, a.bias_down = (_ptr(b) for b in self.biases)
        if act == "swigluoai" or any(b is not None for b in self.biases):
            a.T_max, a.H, a.I, a.E, a.B, a.topk = T_max, self.H, self.I, E, B, topk
            a.w_gate, a.act, a.act_quant = w_gate.desc, self.act, act_quant
            n = _lib.moe_forward_workspace_size_args(ctypes.byref(a))
            self.ws = torch.zeros(n, dtype=torch.uint8, device=w_gate.data.device)
        else:
            self.ws = forward_workspace(T_max, self.H, self.I, E, B, topk, w_gate.fmt, act_quant,
                                        w_gate.data.device)
        self.args.routing = ROUTING[routing]
        self.routing_bias = routing_bias
        self.args.n_group, self.args.topk_group = n_group, topk_group
        self.args.routed_scaling_factor = routed_scaling_factor
        self.args.apply_router_weight_on_input = 1 if apply_router_weight_on_input else 0

    def __call__(self, x, router_logits=None, out=None, topk_ids=None, topk_w=None, stream=None,
                 stage_events=None, topk_ids_in=None, topk_w_in=None):
        """``stage_events``: None, or a list of MOE_FWD_STAGE_EVENTS entries, each None (not
        recorded) or a torch.cuda.Event created with enable_timing and recorded once (so that
        its handle exists). ``topk_ids_in``/``topk_w_in``: the given top-k of routing "given"."""
        T = x.shape[0]
        if stage_events is not None:
            if len(stage_events) != MOE_FWD_STAGE_EVENTS:
                raise ValueError(f"need {MOE_FWD_STAGE_EVENTS} events")
            self._ev = (ctypes.c_void_p * MOE_FWD_STAGE_EVENTS)(
                *[None if e is None else e.cuda_event for e in stage_events])
            self.args.stage_events = ctypes.cast(self._ev, ctypes.c_void_p)
        else:
            self.args.stage_events = None
        out = out if out is not None else torch.empty(T, self.H, dtype=torch.bfloat16, device=x.device)
        a = self.args
        a.x, a.router_logits = _ptr(x), _ptr(router_logits)
        a.T, a.H, a.I, a.E, a.B, a.topk = T, self.H, self.I, self.E, self.B, self.topk
        a.replica_src = _ptr(self.replica_src)
        a.w_gate, a.w_up, a.w_down = self.w_gate.desc, self.w_up.desc, self.w_down.desc
        a.act = self.act
        a.apply_topk_in_fc1 = 1 if self.apply_topk_in_fc1 else 0
        a.act_quant = self.act_quant
        a.out = _ptr(out)
        a.topk_ids_out, a.topk_w_out = _ptr(topk_ids), _ptr(topk_w)
        a.T_max = self.T_max
        a.routing_bias = _ptr(self.routing_bias)
        a.topk_ids_in, a.topk_w_in = _ptr(topk_ids_in), _ptr(topk_w_in)
        _check(_lib.moe_forward(ctypes.byref(a), _ptr(self.ws), self.ws.numel(), _stream(stream)),
               "moe_forward")
        return out

    def device_error(self, stream=None) -> int:
        return _lib.moe_get_device_error(_ptr(self.ws), _stream(stream))

    def graph(self, x, router_logits=None, out=None, warmup: int = 1, **kw):
        """One forward on these buffers captured into a CUDA graph; ``graph.replay()`` reruns the
        layer on whatever x / router_logits (and the given top-k, if any) then hold and writes
        ``out``. ``warmup`` eager calls on a side stream come first: they also set the library's
        one-time host state (kernel attributes, the SM count), which must not be set up during
        capture. Returns ``(graph, out)``."""
        T = x.shape[0]
        out = out if out is not None else torch.empty(T, self.H, dtype=torch.bfloat16, device=x.device)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(warmup):
                self(x, router_logits, out=out, **kw)
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self(x, router_logits, out=out, **kw)
        return g, out


def moe_forward(x, router_logits, w_gate: Weight, w_up: Weight, w_down: Weight, E: int, topk: int,
                B: int = 0, replica_src=None, act="silu", situ_alpha=1.0, situ_beta=1.0, act_quant=0,
                apply_topk_in_fc1=True, topk_ids=None, topk_w=None):
    layer = MoEForward(w_gate, w_up, w_down, E, topk, B, replica_src, act, situ_alpha, situ_beta,
                       act_quant, apply_topk_in_fc1, T_max=max(1, x.shape[0]))
    out = layer(x, router_logits, topk_ids=topk_ids, topk_w=topk_w)
    return out, layer


def moe_get_device_error(ws: torch.Tensor, stream=None) -> int:
    return _lib.moe_get_device_error(_ptr(ws), _stream(stream))
