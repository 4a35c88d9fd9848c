"""One MoE layer step (forward + backward) through the C ABI, with every
buffer allocated once up front so that a step allocates nothing."""
from __future__ import annotations

import torch

from . import binding as B


class MoELayerStep:
    """Buffers and call sequence of one forward+backward pass.

    forward(): moe_route -> moe_permute -> moe_expert_ffn_fwd -> moe_combine
    backward(): moe_layer_bwd (saved set: x, logits, idx, gate, plan, H)
    """

    def __init__(self, T, d, f, E, k, dtype=torch.bfloat16, device="cuda",
                 round_mode=B.MOE_ROUND_NONE, balance_lambda=None,
                 gate_mode=B.MOE_GATE_TOPK_SOFTMAX, capacity_factor=None, precision="bf16",
                 mx_wgrad=False):
        self.T, self.d, self.f, self.E, self.k = T, d, f, E, k
        self.dtype, self.device, self.round_mode = dtype, device, round_mode
        self.gate_mode = gate_mode
        if precision not in ("bf16", "mxfp8"):
            raise ValueError("precision must be 'bf16' or 'mxfp8'")
        self.precision = precision
        self.mx_wgrad = bool(mx_wgrad) and precision == "mxfp8"
        if round_mode == B.MOE_ROUND_CAPACITY:
            if capacity_factor is None:
                raise ValueError("MOE_ROUND_CAPACITY needs capacity_factor")
            self.capacity = B.capacity_from_factor(T, E, k, capacity_factor)
        else:
            self.capacity = -1
        dt = B.dtype_code(dtype)
        cap = B.moe_row_capacity(T, E, k)
        self.cap = cap
        e = lambda *s, dt_=torch.float32: torch.empty(*s, device=device, dtype=dt_)
        self.logits, self.idx, self.gate = e(T, E), e(T, k, dt_=torch.int32), e(T, k)
        self.plan = dict(counts=e(E, dt_=torch.int32), offsets=e(E + 1, dt_=torch.int32),
                         row_token=e(cap, dt_=torch.int32), row_gate=e(cap),
                         row_slot=e(cap, dt_=torch.int32), slot_row=e(T * k, dt_=torch.int32),
                         extra_row=e(T, E, dt_=torch.int32)
                         if round_mode == B.MOE_ROUND_NEAREST else None)
        self.H, self.Y = e(cap, 2 * f, dt_=dtype), e(cap, d, dt_=dtype)
        self.out = e(T, d, dt_=dtype)
        self.ws_perm = e(max(B.moe_permute_workspace_size(T, E, k, round_mode), 1), dt_=torch.uint8)
        if precision == "mxfp8":
            self.wq = {n: e(sz, dt_=torch.uint8) for n, sz in
                       zip(B.MX_WEIGHT_NAMES, B.moe_mxfp8_weight_sizes(E, d, f))}
            self.ws_mx = e(max(B.moe_ffn_fwd_mxfp8_workspace_size(T, d, f, E, k), 1),
                           dt_=torch.uint8)
            self.ws_bwd = e(max(B.moe_layer_bwd_mxfp8_workspace_size(T, d, f, E, k,
                                                                     self.mx_wgrad), 1),
                            dt_=torch.uint8)
        else:
            self.ws_fwd = e(max(B.moe_ffn_fwd_workspace_size(T, d, f, E, k, dt), 1),
                            dt_=torch.uint8)
            self.ws_bwd = e(max(B.moe_layer_bwd_workspace_size(T, d, f, E, k, dt), 1),
                            dt_=torch.uint8)
        self.balance_lambda = balance_lambda
        if balance_lambda is not None:
            self.ws_bal = e(max(B.lib().moe_balance_loss_workspace_size(T, E, k), 1), dt_=torch.uint8)
        self.balance = None
        self.grads = dict(dx=e(T, d, dt_=dtype), dw_gate=e(d, E), dw1=e(E, d, f, dt_=dtype),
                          dw3=e(E, d, f, dt_=dtype), dw2=e(E, f, d, dt_=dtype), dS=e(cap),
                          dlogits=e(T, E))

    def forward(self, x, w_gate, w1, w3, w2, logits_override=None, logit_bias=None, stream=None,
                logit_noise=None):
        self._saved = (x, w_gate, w1, w3, w2)
        self.router_grad = logits_override is None
        B.moe_route(x, w_gate, self.k, logits_override, logit_bias, self.logits, self.idx,
                    self.gate, T=self.T, E=self.E, stream=stream, gate_mode=self.gate_mode,
                    logit_noise=logit_noise)
        B.moe_permute(self.idx, self.gate, self.logits, self.E, self.round_mode, out=self.plan,
                      ws=self.ws_perm, stream=stream, gate_mode=self.gate_mode,
                      capacity=self.capacity)
        if self.balance_lambda is not None:
            self.balance = B.moe_balance_loss(self.idx, self.gate, self.E, self.balance_lambda,
                                              ws=self.ws_bal, stream=stream)
        if self.precision == "mxfp8":
            # weights change every optimizer step: quantise them in the step
            B.moe_mxfp8_quantize_weights(w1, w3, w2, out=self.wq, stream=stream)
            B.moe_expert_ffn_fwd_mxfp8(x, self.wq, self.plan, self.k, self.E, self.f, self.H,
                                       self.Y, self.ws_mx, stream=stream)
        else:
            B.moe_expert_ffn_fwd(x, w1, w3, w2, self.plan, self.k, self.H, self.Y, self.ws_fwd,
                                 stream=stream)
        B.moe_combine(self.Y, self.plan["row_gate"], self.plan["slot_row"],
                      self.plan["extra_row"], self.T, self.E, self.k, self.out, stream=stream)
        return self.out

    def capture(self, x, w_gate, w1, w3, w2, dout, logits_override=None, logit_bias=None,
                logit_noise=None):
        """Record one forward + backward step into a CUDA graph and return it.

        Every library call only enqueues kernels on the current stream (no host
        synchronisation, no allocation), so the whole step can be captured;
        ``graph.replay()`` then re-runs it on the current contents of the given
        tensors and of this object's buffers.  One eager step first (on a side
        stream) sets the kernels' shared-memory attributes outside capture."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.forward(x, w_gate, w1, w3, w2, logits_override, logit_bias, logit_noise=logit_noise)
            self.backward(dout)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            self.forward(x, w_gate, w1, w3, w2, logits_override, logit_bias, logit_noise=logit_noise)
            self.backward(dout)
        return graph

    def backward(self, dout, stream=None):
        x, w_gate, w1, w3, w2 = self._saved
        gate_grad = self.balance["dgate"] if self.balance else None
        if self.precision == "mxfp8":   # dX (and with mx_wgrad the dW) GEMMs on MXFP8 operands
            return B.moe_layer_bwd_mxfp8(dout, x, w_gate, w1, w3, w2, self.wq, self.idx,
                                         self.gate, self.plan, self.H, self.router_grad,
                                         out=self.grads, ws=self.ws_bwd, stream=stream,
                                         gate_grad=gate_grad, logits=self.logits,
                                         gate_mode=self.gate_mode, wgrad=self.mx_wgrad)
        return B.moe_layer_bwd(dout, x, w_gate, w1, w3, w2, self.idx, self.gate, self.plan,
                               self.H, self.router_grad, out=self.grads, ws=self.ws_bwd,
                               stream=stream, gate_grad=gate_grad, logits=self.logits,
                               gate_mode=self.gate_mode)
