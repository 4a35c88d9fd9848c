"""Python binding of ``libmoe_b200.so`` (ctypes; argument marshalling only).

Every function here has the name of the C entry point it calls and does
nothing but turn torch tensors into device pointers, allocate outputs the
caller did not pass, and raise ``MoEError`` on a non-zero return code.  All
arithmetic happens in the library's CUDA kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_F32, MOE_BF16 = 0, 1
MOE_ROUND_NONE, MOE_ROUND_NEAREST, MOE_ROUND_CAPACITY = 0, 1, 2
MOE_GATE_TOPK_SOFTMAX, MOE_GATE_SOFTMAX_TOPK = 0, 1
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA = 0, -1, -2, -3
MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_WORKSPACE, MOE_ERR_DEVICE_CHECK = -4, -5, -6
TILE = 128

EXPORTS = [
    "moe_version", "moe_last_error", "moe_row_capacity", "moe_route",
    "moe_permute_workspace_size", "moe_permute", "moe_ffn_fwd_workspace_size",
    "moe_expert_ffn_fwd", "moe_combine", "moe_layer_bwd_workspace_size", "moe_layer_bwd",
    "moe_check_status", "moe_profile_enable", "moe_profile_report", "moe_permute_noalloc",
    "moe_balance_loss_workspace_size", "moe_balance_loss",
    "moe_mxfp8_weight_sizes", "moe_mxfp8_quantize_weights", "moe_ffn_fwd_mxfp8_workspace_size",
    "moe_mxfp8_quantize_tokens",
    "moe_expert_ffn_fwd_mxfp8", "moe_layer_bwd_mxfp8_workspace_size", "moe_layer_bwd_mxfp8",
    "moe_debug_expire_next_wait", "moe_gather_rows", "moe_ep_dispatch_counts",
    "moe_ep_receive_plan", "moe_expert_rows_fwd_workspace_size", "moe_expert_rows_fwd",
    "moe_expert_rows_bwd_workspace_size", "moe_expert_rows_bwd", "moe_token_bwd_workspace_size",
    "moe_token_bwd",
]

_lib = None


class MoEError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"moe error {code}: {msg}")
        self.code = code


_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t

_SIGS = {
    "moe_version": (_i, []),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_row_capacity": (_sz, [_i, _i, _i, _i]),
    "moe_route": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_permute_workspace_size": (_sz, [_i, _i, _i, _i]),
    "moe_permute": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp,
                         _vp, _vp, _vp, _sz, _vp]),
    "moe_ffn_fwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "moe_expert_ffn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                _vp, _vp, _vp, _sz, _vp]),
    "moe_combine": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp]),
    "moe_layer_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "moe_layer_bwd": (_i, [_vp] * 10 + [_i] + [_vp] * 6 + [_i] * 7 + [_vp] * 7 + [_vp, _sz, _vp]),
    "moe_balance_loss_workspace_size": (_sz, [_i, _i, _i]),
    "moe_balance_loss": (_i, [_vp, _vp, _i, _i, _i, ctypes.c_float, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_mxfp8_weight_sizes": (_i, [_i, _i, _i, ctypes.POINTER(_sz)]),
    "moe_mxfp8_quantize_weights": (_i, [_vp, _vp, _vp, _i, _i, _i] + [_vp] * 9),
    "moe_mxfp8_quantize_tokens": (_i, [_vp, _i, _vp, _vp, _i, _i, _i, _vp, _vp, _vp]),
    "moe_layer_bwd_mxfp8_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "moe_layer_bwd_mxfp8": (_i, [_vp] * 14 + [_i] + [_vp] * 6 + [_i] * 7 + [_vp] * 8 + [_sz, _vp]),
    "moe_ffn_fwd_mxfp8_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "moe_expert_ffn_fwd_mxfp8": (_i, [_vp] * 9 + [_i] * 5 + [_vp, _vp, _vp, _sz, _vp]),
    "moe_check_status": (_i, [_vp]),
    "moe_profile_enable": (_i, [_i]),
    "moe_permute_noalloc": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_profile_report": (_i, [ctypes.c_char_p, _sz]),
    "moe_debug_expire_next_wait": (_i, [ctypes.c_longlong]),
    "moe_gather_rows": (_i, [_vp] * 5 + [_i] * 5 + [_vp, _vp]),
    "moe_ep_dispatch_counts": (_i, [_vp, _i, _vp, _vp]),
    "moe_ep_receive_plan": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
    "moe_expert_rows_fwd_workspace_size": (_sz, [_i, _i, _i]),
    "moe_expert_rows_fwd": (_i, [_vp] * 5 + [_i] * 5 + [_vp] * 3 + [_sz, _vp]),
    "moe_expert_rows_bwd_workspace_size": (_sz, [_i] * 4),
    "moe_expert_rows_bwd": (_i, [_vp] * 8 + [_i] * 5 + [_vp] * 6 + [_sz, _vp]),
    "moe_token_bwd_workspace_size": (_sz, [_i] * 5),
    "moe_token_bwd": (_i, [_vp] * 8 + [_i] + [_vp] * 3 + [_i] * 6 + [_vp] * 4 + [_sz, _vp]),
}


def lib() -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m mixture_experts_layer_59_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc):
    if rc != 0:
        raise MoEError(rc, lib().moe_last_error().decode())


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return MOE_BF16
    if dt == torch.float32:
        return MOE_F32
    raise ValueError(f"unsupported dtype {dt}")


def moe_version() -> int:
    return lib().moe_version()


def moe_row_capacity(T, E, k, tile=TILE) -> int:
    return lib().moe_row_capacity(T, E, k, tile)


def moe_route(x, w_gate, k, logits_override=None, logit_bias=None, logits=None, idx=None,
              gate=None, T=None, E=None, stream=None, gate_mode=MOE_GATE_TOPK_SOFTMAX,
              logit_noise=None):
    """logits [T,E] f32, idx [T,k] i32, gate [T,k] f32 (outputs allocated if None).
    gate_mode: MOE_GATE_TOPK_SOFTMAX (softmax over the k chosen logits) or
    MOE_GATE_SOFTMAX_TOPK (softmax over all E, the k largest kept).
    logit_noise [T,E] f32: routing noise added to the scores (noisy top-k)."""
    if T is None:
        T = (logits_override if logits_override is not None else x).shape[0]
    if E is None:
        E = (logits_override if logits_override is not None else w_gate).shape[1]
    dev = (logits_override if logits_override is not None else x).device
    d = x.shape[1] if x is not None else 0
    dt = dtype_code(x.dtype) if x is not None else MOE_F32
    logits = logits if logits is not None else torch.empty(T, E, device=dev, dtype=torch.float32)
    idx = idx if idx is not None else torch.empty(T, k, device=dev, dtype=torch.int32)
    gate = gate if gate is not None else torch.empty(T, k, device=dev, dtype=torch.float32)
    _check(lib().moe_route(_p(x), _p(w_gate), T, d, E, k, dt, gate_mode, _p(logits_override),
                           _p(logit_bias), _p(logit_noise),
                           _p(logits), _p(idx), _p(gate), _stream(stream)))
    return logits, idx, gate


def moe_permute_workspace_size(T, E, k, round_mode) -> int:
    return lib().moe_permute_workspace_size(T, E, k, round_mode)


def capacity_from_factor(T, E, k, factor) -> int:
    """Tokens per expert for a capacity factor: ceil(factor * T * k / E)."""
    return int(math.ceil(factor * T * k / E))


def moe_permute(idx, gate, logits, E, round_mode=MOE_ROUND_NONE, tile=TILE, out=None, ws=None,
                stream=None, gate_mode=MOE_GATE_TOPK_SOFTMAX, capacity=-1):
    """Returns dict counts, offsets, row_token, row_gate, row_slot, slot_row, extra_row
    (extra_row only with MOE_ROUND_NEAREST, else None).  capacity: tokens per
    expert with MOE_ROUND_CAPACITY."""
    T, k = idx.shape
    dev = idx.device
    cap = moe_row_capacity(T, E, k, tile)
    o = dict(out) if out else {}
    o.setdefault("counts", torch.empty(E, device=dev, dtype=torch.int32))
    o.setdefault("offsets", torch.empty(E + 1, device=dev, dtype=torch.int32))
    o.setdefault("row_token", torch.empty(cap, device=dev, dtype=torch.int32))
    o.setdefault("row_gate", torch.empty(cap, device=dev, dtype=torch.float32))
    o.setdefault("row_slot", torch.empty(cap, device=dev, dtype=torch.int32))
    o.setdefault("slot_row", torch.empty(T * k, device=dev, dtype=torch.int32))
    if round_mode == MOE_ROUND_NEAREST:
        o.setdefault("extra_row", torch.empty(T, E, device=dev, dtype=torch.int32))
    else:
        o.setdefault("extra_row", None)
    wsb = moe_permute_workspace_size(T, E, k, round_mode)
    if ws is None:
        ws = torch.empty(max(wsb, 1), device=dev, dtype=torch.uint8)
    _check(lib().moe_permute(_p(idx), _p(gate), _p(logits), T, E, k, round_mode, tile,
                             gate_mode, capacity,
                             _p(o["counts"]), _p(o["offsets"]), _p(o["row_token"]),
                             _p(o["row_gate"]), _p(o["row_slot"]), _p(o["slot_row"]),
                             _p(o["extra_row"]), _p(ws), ws.numel(), _stream(stream)))
    return o


def moe_ffn_fwd_workspace_size(T, d, f, E, k, dtype) -> int:
    return lib().moe_ffn_fwd_workspace_size(T, d, f, E, k, dtype)


def moe_expert_ffn_fwd(x, w1, w3, w2, plan, k, H=None, Y_perm=None, ws=None, stream=None):
    """plan: dict from moe_permute (row_token, offsets, slot_row, extra_row)."""
    T, d = x.shape
    E, _, f = w1.shape
    dt = dtype_code(x.dtype)
    cap = moe_row_capacity(T, E, k)
    H = H if H is not None else torch.empty(cap, 2 * f, device=x.device, dtype=x.dtype)
    Y_perm = Y_perm if Y_perm is not None else torch.empty(cap, d, device=x.device, dtype=x.dtype)
    if ws is None:
        ws = torch.empty(max(moe_ffn_fwd_workspace_size(T, d, f, E, k, dt), 1), device=x.device,
                         dtype=torch.uint8)
    _check(lib().moe_expert_ffn_fwd(_p(x), _p(w1), _p(w3), _p(w2), _p(plan["row_token"]),
                                    _p(plan["offsets"]), _p(plan["slot_row"]),
                                    _p(plan.get("extra_row")), T, d, f, E, k, dt, _p(H),
                                    _p(Y_perm), _p(ws), ws.numel(), _stream(stream)))
    return H, Y_perm


MX_WEIGHT_NAMES = ("w13q", "w13s", "w2q", "w2s", "w1rq", "w1rs", "w3rq", "w3rs")


def moe_mxfp8_weight_sizes(E, d, f):
    """Bytes of (W13q, W13s, W2q, W2s, W1r, W1r scales, W3r, W3r scales)."""
    sz = (_sz * 8)()
    _check(lib().moe_mxfp8_weight_sizes(E, d, f, sz))
    return tuple(int(v) for v in sz)


def moe_mxfp8_quantize_tokens(src, offsets, capr, gather_row=None, stream=None):
    """Row-space matrix quantised along its rows (blocks of 32 rows): returns
    (q [n, capr] uint8 E4M3, sf uint8 scales) for the rows below offsets[E]."""
    n = src.shape[1]
    E = offsets.numel() - 1
    q = torch.zeros(n, capr, device=src.device, dtype=torch.uint8)
    sf = torch.zeros(n * capr // 32, device=src.device, dtype=torch.uint8)
    _check(lib().moe_mxfp8_quantize_tokens(_p(src), src.shape[0], _p(gather_row), _p(offsets), E,
                                           n, capr, _p(q), _p(sf), _stream(stream)))
    return q, sf


def moe_mxfp8_quantize_weights(w1, w3, w2, out=None, stream=None, backward=True):
    """MXFP8 copies of the expert weights: dict w13q, w13s, w2q, w2s and, with
    ``backward``, w1rq, w1rs, w3rq, w3rs (for moe_layer_bwd_mxfp8); uint8."""
    E, d, f = w1.shape
    o = dict(out) if out else {}
    names = MX_WEIGHT_NAMES if backward else MX_WEIGHT_NAMES[:4]
    for name, n in zip(names, moe_mxfp8_weight_sizes(E, d, f)):
        o.setdefault(name, torch.empty(n, device=w1.device, dtype=torch.uint8))
    r = [_p(o.get(n)) if backward else None for n in MX_WEIGHT_NAMES[4:]]
    _check(lib().moe_mxfp8_quantize_weights(_p(w1), _p(w3), _p(w2), E, d, f, _p(o["w13q"]),
                                            _p(o["w13s"]), _p(o["w2q"]), _p(o["w2s"]), *r,
                                            _stream(stream)))
    return o


def moe_ffn_fwd_mxfp8_workspace_size(T, d, f, E, k) -> int:
    return lib().moe_ffn_fwd_mxfp8_workspace_size(T, d, f, E, k)


def moe_expert_ffn_fwd_mxfp8(x, wq, plan, k, E, f, H=None, Y_perm=None, ws=None, stream=None):
    """MXFP8 forward of the expert FFN.  wq: dict from moe_mxfp8_quantize_weights."""
    T, d = x.shape
    cap = moe_row_capacity(T, E, k)
    H = H if H is not None else torch.empty(cap, 2 * f, device=x.device, dtype=x.dtype)
    Y_perm = Y_perm if Y_perm is not None else torch.empty(cap, d, device=x.device, dtype=x.dtype)
    if ws is None:
        ws = torch.empty(max(moe_ffn_fwd_mxfp8_workspace_size(T, d, f, E, k), 1), device=x.device,
                         dtype=torch.uint8)
    _check(lib().moe_expert_ffn_fwd_mxfp8(
        _p(x), _p(wq["w13q"]), _p(wq["w13s"]), _p(wq["w2q"]), _p(wq["w2s"]), _p(plan["row_token"]),
        _p(plan["offsets"]), _p(plan["slot_row"]), _p(plan.get("extra_row")), T, d, f, E, k,
        _p(H), _p(Y_perm), _p(ws), ws.numel(), _stream(stream)))
    return H, Y_perm


def moe_combine(Y_perm, row_gate, slot_row, extra_row, T, E, k, out=None, stream=None):
    d = Y_perm.shape[1]
    out = out if out is not None else torch.empty(T, d, device=Y_perm.device, dtype=Y_perm.dtype)
    _check(lib().moe_combine(_p(Y_perm), _p(row_gate), _p(slot_row), _p(extra_row), T, d, E, k,
                             dtype_code(Y_perm.dtype), _p(out), _stream(stream)))
    return out


def moe_layer_bwd_workspace_size(T, d, f, E, k, dtype) -> int:
    return lib().moe_layer_bwd_workspace_size(T, d, f, E, k, dtype)


def moe_layer_bwd(dout, x, w_gate, w1, w3, w2, idx, gate, plan, H, router_grad=True, out=None,
                  ws=None, stream=None, gate_grad=None, logits=None,
                  gate_mode=MOE_GATE_TOPK_SOFTMAX):
    """plan: dict from moe_permute.  Returns dict dx, dw_gate, dw1, dw3, dw2, dS, dlogits.
    logits (from moe_route) are needed with MOE_GATE_SOFTMAX_TOPK."""
    T, d = x.shape
    E, _, f = w1.shape
    k = idx.shape[1]
    dt = dtype_code(x.dtype)
    cap = moe_row_capacity(T, E, k)
    dev = x.device
    o = dict(out) if out else {}
    o.setdefault("dx", torch.empty(T, d, device=dev, dtype=x.dtype))
    o.setdefault("dw_gate", torch.empty(d, E, device=dev, dtype=torch.float32))
    o.setdefault("dw1", torch.empty_like(w1))
    o.setdefault("dw3", torch.empty_like(w3))
    o.setdefault("dw2", torch.empty_like(w2))
    o.setdefault("dS", torch.empty(cap, device=dev, dtype=torch.float32))
    o.setdefault("dlogits", torch.empty(T, E, device=dev, dtype=torch.float32))
    if ws is None:
        ws = torch.empty(max(moe_layer_bwd_workspace_size(T, d, f, E, k, dt), 1), device=dev,
                         dtype=torch.uint8)
    _check(lib().moe_layer_bwd(
        _p(dout), _p(x), _p(w_gate), _p(w1), _p(w3), _p(w2), _p(idx), _p(gate), _p(gate_grad),
        _p(logits), gate_mode, _p(plan["offsets"]), _p(plan["row_token"]), _p(plan["row_gate"]), _p(plan["slot_row"]),
        _p(plan.get("extra_row")), _p(H), T, d, f, E, k, dt, 1 if router_grad else 0,
        _p(o["dx"]), _p(o["dw_gate"]), _p(o["dw1"]), _p(o["dw3"]), _p(o["dw2"]), _p(o["dS"]),
        _p(o["dlogits"]), _p(ws), ws.numel(), _stream(stream)))
    return o


def moe_layer_bwd_mxfp8_workspace_size(T, d, f, E, k, wgrad=False) -> int:
    return lib().moe_layer_bwd_mxfp8_workspace_size(T, d, f, E, k, 1 if wgrad else 0)


def moe_layer_bwd_mxfp8(dout, x, w_gate, w1, w3, w2, wq, idx, gate, plan, H, router_grad=True,
                        out=None, ws=None, stream=None, gate_grad=None, logits=None,
                        gate_mode=MOE_GATE_TOPK_SOFTMAX, wgrad=False):
    """moe_layer_bwd with the dX GEMM on MXFP8 operands, and with wgrad the
    weight-gradient GEMMs too.  wq: dict from moe_mxfp8_quantize_weights
    (backward=True)."""
    T, d = x.shape
    E, _, f = w1.shape
    k = idx.shape[1]
    cap = moe_row_capacity(T, E, k)
    dev = x.device
    o = dict(out) if out else {}
    o.setdefault("dx", torch.empty(T, d, device=dev, dtype=x.dtype))
    o.setdefault("dw_gate", torch.empty(d, E, device=dev, dtype=torch.float32))
    o.setdefault("dw1", torch.empty_like(w1))
    o.setdefault("dw3", torch.empty_like(w3))
    o.setdefault("dw2", torch.empty_like(w2))
    o.setdefault("dS", torch.empty(cap, device=dev, dtype=torch.float32))
    o.setdefault("dlogits", torch.empty(T, E, device=dev, dtype=torch.float32))
    if ws is None:
        ws = torch.empty(max(moe_layer_bwd_mxfp8_workspace_size(T, d, f, E, k, wgrad), 1),
                         device=dev, dtype=torch.uint8)
    _check(lib().moe_layer_bwd_mxfp8(
        _p(dout), _p(x), _p(w_gate), _p(w1), _p(w3), _p(w2), _p(wq["w1rq"]), _p(wq["w1rs"]),
        _p(wq["w3rq"]), _p(wq["w3rs"]), _p(idx), _p(gate), _p(gate_grad), _p(logits), gate_mode,
        _p(plan["offsets"]), _p(plan["row_token"]), _p(plan["row_gate"]), _p(plan["slot_row"]),
        _p(plan.get("extra_row")), _p(H), T, d, f, E, k, 1 if router_grad else 0,
        1 if wgrad else 0,
        _p(o["dx"]), _p(o["dw_gate"]), _p(o["dw1"]), _p(o["dw3"]), _p(o["dw2"]), _p(o["dS"]),
        _p(o["dlogits"]), _p(ws), ws.numel(), _stream(stream)))
    return o


def moe_check_status(stream=None):
    _check(lib().moe_check_status(_stream(stream)))


def moe_profile_enable(on: bool = True):
    _check(lib().moe_profile_enable(1 if on else 0))


def moe_profile_report() -> dict:
    """{kernel name: (launches, total_ms, median_ms)} of the launches recorded
    since the last report (waits for their events); median_ms is the median
    time of one launch."""
    buf = ctypes.create_string_buffer(1 << 16)
    _check(lib().moe_profile_report(buf, len(buf)))
    out = {}
    for line in buf.value.decode().splitlines():
        name, n, ms, med = line.split()
        out[name] = (int(n), float(ms), float(med))
    return out


def moe_permute_noalloc(idx, gate, E, tile=TILE, out=None, stream=None):
    """moe_permute without rounding and without a workspace (static device
    scratch, T <= 65536).  Output buffers are allocated here if not passed."""
    T, k = idx.shape
    dev = idx.device
    cap = moe_row_capacity(T, E, k, tile)
    o = dict(out) if out else {}
    o.setdefault("counts", torch.empty(E, device=dev, dtype=torch.int32))
    o.setdefault("offsets", torch.empty(E + 1, device=dev, dtype=torch.int32))
    o.setdefault("row_token", torch.empty(cap, device=dev, dtype=torch.int32))
    o.setdefault("row_gate", torch.empty(cap, device=dev, dtype=torch.float32))
    o.setdefault("row_slot", torch.empty(cap, device=dev, dtype=torch.int32))
    o.setdefault("slot_row", torch.empty(T * k, device=dev, dtype=torch.int32))
    o.setdefault("extra_row", None)
    _check(lib().moe_permute_noalloc(_p(idx), _p(gate), T, E, k, tile, _p(o["counts"]),
                                     _p(o["offsets"]), _p(o["row_token"]), _p(o["row_gate"]),
                                     _p(o["row_slot"]), _p(o["slot_row"]), _stream(stream)))
    return o


def moe_balance_loss(idx, gate, E, lam, dgate=True, ws=None, stream=None):
    """Returns dict(stats [4] = loss, max share, count CV^2, count MSE;
    importance [E]; dgate [T,k] or None)."""
    T, k = idx.shape
    dev = idx.device
    stats = torch.empty(4, device=dev, dtype=torch.float32)
    imp = torch.empty(E, device=dev, dtype=torch.float32)
    dg = torch.empty(T, k, device=dev, dtype=torch.float32) if dgate else None
    if ws is None:
        ws = torch.empty(max(lib().moe_balance_loss_workspace_size(T, E, k), 1), device=dev,
                         dtype=torch.uint8)
    _check(lib().moe_balance_loss(_p(idx), _p(gate), T, E, k, float(lam), _p(stats), _p(imp),
                                  _p(dg), _p(ws), ws.numel(), _stream(stream)))
    return dict(stats=stats, importance=imp, dgate=dg)


# ------------------------------------------------------------------ expert parallelism
def moe_gather_rows(src, plan, k, out=None, stream=None):
    """Rows of a plan gathered from token-major ``src`` [T, width]; padding rows zero."""
    T, width = src.shape
    E = plan["offsets"].numel() - 1
    cap = moe_row_capacity(T, E, k)
    out = out if out is not None else torch.empty(cap, width, device=src.device, dtype=src.dtype)
    _check(lib().moe_gather_rows(_p(src), _p(plan["row_token"]), _p(plan["offsets"]),
                                 _p(plan["slot_row"]), _p(plan.get("extra_row")), T, width, E, k,
                                 dtype_code(src.dtype), _p(out), _stream(stream)))
    return out


def moe_ep_dispatch_counts(offsets, out=None, stream=None):
    """Rows of each expert's segment [E] (int32, device)."""
    E = offsets.numel() - 1
    out = out if out is not None else torch.empty(E, device=offsets.device, dtype=torch.int32)
    _check(lib().moe_ep_dispatch_counts(_p(offsets), E, _p(out), _stream(stream)))
    return out


def moe_ep_receive_plan(recv_rows, stream=None):
    """recv_rows [G, El] int32 -> (local_offsets [El+1], recv_row [G, El])."""
    G, El = recv_rows.shape
    lo = torch.empty(El + 1, device=recv_rows.device, dtype=torch.int32)
    rr = torch.empty(G, El, device=recv_rows.device, dtype=torch.int32)
    _check(lib().moe_ep_receive_plan(_p(recv_rows), G, El, _p(lo), _p(rr), _stream(stream)))
    return lo, rr


def moe_expert_rows_fwd(xg, w1, w3, w2, offsets, H=None, Y=None, ws=None, stream=None):
    """Grouped SwiGLU FFN on expert-contiguous rows: H [rows, 2f], Y [rows, d]."""
    rows, d = xg.shape
    E, _, f = w1.shape
    dt = dtype_code(xg.dtype)
    H = H if H is not None else torch.empty(rows, 2 * f, device=xg.device, dtype=xg.dtype)
    Y = Y if Y is not None else torch.empty(rows, d, device=xg.device, dtype=xg.dtype)
    if ws is None:
        ws = torch.empty(max(lib().moe_expert_rows_fwd_workspace_size(rows, f, dt), 1),
                         device=xg.device, dtype=torch.uint8)
    _check(lib().moe_expert_rows_fwd(_p(xg), _p(w1), _p(w3), _p(w2), _p(offsets), rows, d, f, E,
                                     dt, _p(H), _p(Y), _p(ws), ws.numel(), _stream(stream)))
    return H, Y


def moe_expert_rows_bwd(dog, xg, row_gate, H, w1, w3, w2, offsets, out=None, ws=None,
                        stream=None):
    """Expert side of the backward on expert-contiguous rows.  Returns dict
    dX_rows [rows, d], dS [rows] f32, dw1, dw3 [E, d, f], dw2 [E, f, d]."""
    rows, d = xg.shape
    E, _, f = w1.shape
    dt = dtype_code(xg.dtype)
    dev = xg.device
    o = dict(out) if out else {}
    o.setdefault("dX_rows", torch.empty(rows, d, device=dev, dtype=xg.dtype))
    o.setdefault("dS", torch.empty(rows, device=dev, dtype=torch.float32))
    o.setdefault("dw1", torch.empty(E, d, f, device=dev, dtype=xg.dtype))
    o.setdefault("dw3", torch.empty(E, d, f, device=dev, dtype=xg.dtype))
    o.setdefault("dw2", torch.empty(E, f, d, device=dev, dtype=xg.dtype))
    if ws is None:
        ws = torch.empty(max(lib().moe_expert_rows_bwd_workspace_size(rows, d, f, dt), 1),
                         device=dev, dtype=torch.uint8)
    _check(lib().moe_expert_rows_bwd(_p(dog), _p(xg), _p(row_gate), _p(H), _p(w1), _p(w3),
                                     _p(w2), _p(offsets), rows, d, f, E, dt, _p(o["dX_rows"]),
                                     _p(o["dS"]), _p(o["dw1"]), _p(o["dw3"]), _p(o["dw2"]),
                                     _p(ws), ws.numel(), _stream(stream)))
    return o


def moe_token_bwd(dX_rows, dS, x, w_gate, idx, gate, plan, router_grad=True, gate_grad=None,
                  logits=None, gate_mode=MOE_GATE_TOPK_SOFTMAX, out=None, ws=None, stream=None):
    """Token side of the backward.  Returns dict dx [T, d], dw_gate [d, E] f32,
    dlogits [T, E] f32."""
    T, d = x.shape
    k = idx.shape[1]
    E = plan["offsets"].numel() - 1
    dt = dtype_code(x.dtype)
    dev = x.device
    o = dict(out) if out else {}
    o.setdefault("dx", torch.empty(T, d, device=dev, dtype=x.dtype))
    o.setdefault("dw_gate", torch.empty(d, E, device=dev, dtype=torch.float32))
    o.setdefault("dlogits", torch.empty(T, E, device=dev, dtype=torch.float32))
    if ws is None:
        ws = torch.empty(max(lib().moe_token_bwd_workspace_size(T, d, E, k, dt), 1), device=dev,
                         dtype=torch.uint8)
    _check(lib().moe_token_bwd(_p(dX_rows), _p(dS), _p(x), _p(w_gate), _p(idx), _p(gate),
                               _p(gate_grad), _p(logits), gate_mode, _p(plan["row_gate"]),
                               _p(plan["slot_row"]), _p(plan.get("extra_row")), T, d, E, k, dt,
                               1 if router_grad else 0, _p(o["dx"]), _p(o["dw_gate"]),
                               _p(o["dlogits"]), _p(ws), ws.numel(), _stream(stream)))
    return o
