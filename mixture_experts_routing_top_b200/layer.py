"""One MoE layer as a chain of libmoe calls, with every buffer preallocated.

Top-k layer ("MoELayer" of "How MegaDLMs Implements Mixture of Experts (MoE)
Architectures"): route -> permute -> expert MLPs -> unpermute, plus the
shared expert when one is configured.  With a group_of_expert and experts,
the send-once dispatcher of "Expert Coupling in MoE Pretraining" (Abstract):
one row per (token, group) -> the group's local permutation to its experts
-> expert MLPs -> one gate-weighted row per (token, group) -> the token's
sum of its group rows.  Expert-choice layer
("MoELayerExpertChoice"): route_ec -> gather rows -> expert MLPs ->
unpermute_ec.  Nothing here computes: it owns device memory and calls the
library on one stream, with no host synchronisation inside a forward.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import libmoe as M


class TopKLayer:
    def __init__(self, T: int, d: int, E: int, k: int, F: int, capacity_factor: float, dtype: torch.dtype,
                 W1, W3, W2, act: str = "swiglu", norm_topk: bool = False, shared_weights=None,
                 group_of_expert: Optional[torch.Tensor] = None, G: int = 0, out_dtype=None, device="cuda",
                 W_r: Optional[torch.Tensor] = None):
        self.T, self.d, self.E, self.k, self.F = T, d, E, k, F
        self.W_r = W_r                     # router linear gate [E, d]: route from x instead of handed-in logits
        self.cf, self.dtype, self.act, self.norm_topk = capacity_factor, dtype, act, norm_topk
        self.W1, self.W3, self.W2 = W1, W3, W2
        self.goe, self.G = group_of_expert, (G if group_of_expert is not None else 0)
        self.out_dtype = out_dtype or dtype
        dev = torch.device(device)
        self.idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        self.gate = torch.empty((T, k), dtype=torch.float32, device=dev)
        R_max = M.permute_max_rows(T, k, E, capacity_factor, self.G)
        self.R_max = max(R_max, 1)
        self.perm = dict(buffer=torch.empty((self.R_max, d), dtype=dtype, device=dev),
                         row_map=torch.empty((T, k), dtype=torch.int32, device=dev),
                         row_token=torch.empty(self.R_max, dtype=torch.int32, device=dev),
                         counts=torch.empty(E, dtype=torch.int32, device=dev),
                         offsets=torch.empty((self.G or E) + 1, dtype=torch.int32, device=dev),
                         dropped=torch.empty(1, dtype=torch.int32, device=dev))
        self.perm_ws = M._ws(M.permute_workspace_bytes(T, k, E, self.G), dev)
        self.identity = F == 0 or W1 is None
        self.grouped = self.G > 0 and not self.identity
        R_ffn = self.R_max
        if self.grouped:
            # the local expert rows: an indices-only expert-major permute of the same routing
            R_e = max(M.permute_max_rows(T, k, E, capacity_factor, 0), 1)
            self.perm_e = dict(buffer=None, row_map=torch.empty((T, k), dtype=torch.int32, device=dev),
                               row_token=torch.empty(R_e, dtype=torch.int32, device=dev),
                               counts=torch.empty(E, dtype=torch.int32, device=dev),
                               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                               dropped=torch.empty(1, dtype=torch.int32, device=dev))
            self.perm_e_ws = M._ws(M.permute_workspace_bytes(T, k, E, 0), dev)
            self.x_e = torch.empty((R_e, d), dtype=dtype, device=dev)
            self.y_g = torch.empty((self.R_max, d), dtype=dtype, device=dev)
            R_ffn = R_e
        if not self.identity:
            self.y = torch.empty((R_ffn, d), dtype=dtype, device=dev)
            self.ffn_ws = M._ws(M.expert_ffn_workspace_bytes(R_ffn, d, F, dtype), dev)
        self.shared_weights = shared_weights
        if shared_weights is not None:
            sW1 = shared_weights[0]
            self.F_shared = sW1.shape[1]
            self.shared_offsets = torch.tensor([0, T], dtype=torch.int32, device=dev)
            self.shared_y = torch.empty((T, d), dtype=dtype, device=dev)
            self.shared_ws = M._ws(M.expert_ffn_workspace_bytes(T, d, self.F_shared, dtype), dev)
        self.out = torch.empty((T, d), dtype=self.out_dtype, device=dev)

    def route(self, logits, stream=None):
        return M.route_topk(logits, self.k, self.norm_topk, self.idx, self.gate, stream=stream)

    def route_x(self, x, stream=None):
        """The router's linear gate fused with top-k (needs W_r)."""
        return M.router_topk(x, self.W_r, self.k, self.norm_topk, self.idx, self.gate, stream=stream)

    def dispatch(self, x, stream=None):
        p = M.permute(x, self.idx, self.E, self.cf, self.goe, self.G, out=self.perm, workspace=self.perm_ws,
                      stream=stream)
        if self.grouped:
            M.permute(None, self.idx, self.E, self.cf, out=self.perm_e, workspace=self.perm_e_ws, stream=stream)
        return p

    def local_permute(self, stream=None):
        """Group rows -> expert rows (each group's local permutation)."""
        return M.copy_slot_rows(self.perm["buffer"], self.perm["row_map"], self.perm_e["row_map"], self.x_e,
                                stream=stream)

    def expert_mlps(self, stream=None):
        rows, offsets = (self.x_e, self.perm_e["offsets"]) if self.grouped else \
            (self.perm["buffer"], self.perm["offsets"])
        return M.expert_ffn(rows, offsets, self.W1, self.W3, self.W2, self.act, y=self.y, workspace=self.ffn_ws,
                            stream=stream)

    def precombine(self, y, stream=None):
        """Expert outputs -> one gate-weighted row per (token, group)."""
        return M.group_precombine(y, self.perm_e["row_map"], self.perm["row_map"], self.gate, self.y_g,
                                  stream=stream)

    def experts(self, stream=None):
        """Rows the combine reads: the expert outputs, or with groups the
        pre-combined group rows."""
        if self.identity:
            return self.perm["buffer"]
        if not self.grouped:
            return self.expert_mlps(stream)
        self.local_permute(stream)
        return self.precombine(self.expert_mlps(stream), stream)

    def shared_expert(self, x, stream=None):
        if self.shared_weights is None:
            return None
        sW1, sW3, sW2 = self.shared_weights
        return M.expert_ffn(x, self.shared_offsets, sW1, sW3, sW2, "swiglu", y=self.shared_y,
                            workspace=self.shared_ws, stream=stream)

    def combine(self, y, shared=None, stream=None, out=None):
        out = self.out if out is None else out
        if self.grouped:
            return M.unpermute_groups(y, self.perm["row_map"], shared, self.out_dtype, out=out, stream=stream)
        return M.unpermute(y, self.perm["row_map"], self.gate, shared, self.out_dtype, out=out, stream=stream)

    def forward(self, logits: Optional[torch.Tensor], x: torch.Tensor, stream=None, out=None) -> torch.Tensor:
        """logits: the handed-in router logits, or None when the layer has W_r."""
        if self.W_r is not None:
            self.route_x(x, stream)
        else:
            self.route(logits, stream)
        self.dispatch(x, stream)
        y = self.experts(stream)
        sh = self.shared_expert(x, stream)
        return self.combine(y, sh, stream, out)


class ExpertChoiceLayer:
    def __init__(self, T: int, d: int, E: int, C: int, F: int, dtype: torch.dtype, W1, W3, W2, act: str = "gelu",
                 out_dtype=None, device="cuda"):
        self.T, self.d, self.E, self.C, self.F = T, d, E, C, F
        self.dtype, self.act = dtype, act
        self.W1, self.W3, self.W2 = W1, W3, W2
        self.out_dtype = out_dtype or dtype
        dev = torch.device(device)
        R = E * C
        self.R = R
        self.routing = (torch.empty((E, C), dtype=torch.int32, device=dev),
                        torch.empty((E, C), dtype=torch.float32, device=dev),
                        torch.empty(T + 1, dtype=torch.int32, device=dev),
                        torch.empty(R, dtype=torch.int32, device=dev))
        self.route_ws = M._ws(M.route_ec_workspace_bytes(T, E, C), dev)
        self.buffer = torch.empty((R, d), dtype=dtype, device=dev)
        self.offsets = torch.arange(0, R + 1, C, dtype=torch.int32, device=dev)
        self.y = torch.empty((R, d), dtype=dtype, device=dev)
        self.ffn_ws = M._ws(M.expert_ffn_workspace_bytes(R, d, F, dtype), dev)
        self.out = torch.empty((T, d), dtype=self.out_dtype, device=dev)

    def forward(self, logits: torch.Tensor, x: torch.Tensor, stream=None, out=None) -> torch.Tensor:
        ec_token, ec_gate, tok_ptr, tok_row = M.route_ec(logits, self.C, workspace=self.route_ws, out=self.routing,
                                                         stream=stream)
        M.gather_rows(x, tok_ptr, tok_row, self.R, buffer=self.buffer, stream=stream)
        M.expert_ffn(self.buffer, self.offsets, self.W1, self.W3, self.W2, self.act, y=self.y,
                     workspace=self.ffn_ws, stream=stream)
        return M.unpermute_ec(self.y, tok_ptr, tok_row, ec_gate.view(-1), self.out_dtype,
                              out=self.out if out is None else out, stream=stream)


class HostPipeline:
    """Runs a layer over a sequence of batches held in pinned host memory.

    Each batch's inputs are copied to the device on one stream, the layer
    runs on the current stream, and its output is copied back on a third, so
    the copies of batch i+1 and of batch i-1 overlap the compute of batch i.
    Device inputs and outputs are double-buffered; events order every reuse.
    forward(*device_inputs, out=device_output) is the layer call.
    """

    def __init__(self, forward, device_inputs, device_output):
        self.forward = forward
        self.din = [list(device_inputs), [torch.empty_like(t) for t in device_inputs]]
        self.dout = [device_output, torch.empty_like(device_output)]
        self.s_in, self.s_out = torch.cuda.Stream(), torch.cuda.Stream()
        self.ev_in = [torch.cuda.Event() for _ in range(2)]       # inputs landed
        self.ev_used = [torch.cuda.Event() for _ in range(2)]     # compute finished with the inputs
        self.ev_out = [torch.cuda.Event() for _ in range(2)]      # output written
        self.ev_drained = [torch.cuda.Event() for _ in range(2)]  # output copied back

    def run(self, host_inputs, host_outputs):
        """host_inputs[i]: the pinned input tensors of batch i; host_outputs[i]:
        its pinned output tensor.  Returns once everything is enqueued; work
        enqueued on the current stream afterwards runs after the last copy."""
        s_c = torch.cuda.current_stream()
        self.s_in.wait_stream(s_c)
        for i, (hin, hout) in enumerate(zip(host_inputs, host_outputs)):
            b = i & 1
            with torch.cuda.stream(self.s_in):
                if i >= 2:
                    self.s_in.wait_event(self.ev_used[b])
                for h, d in zip(hin, self.din[b]):
                    d.copy_(h, non_blocking=True)
                self.ev_in[b].record(self.s_in)
            s_c.wait_event(self.ev_in[b])
            if i >= 2:
                s_c.wait_event(self.ev_drained[b])
            self.forward(*self.din[b], out=self.dout[b])
            self.ev_used[b].record(s_c)
            self.ev_out[b].record(s_c)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.ev_out[b])
                hout.copy_(self.dout[b], non_blocking=True)
                self.ev_drained[b].record(self.s_out)
        s_c.wait_stream(self.s_out)


class CapturedForward:
    """A layer call captured once into a CUDA graph.

    fn(*inputs, out=out) runs on the current stream with every buffer
    preallocated (the layers here are written that way), so the whole call -
    all its kernels, workspace clears included - can be recorded once and
    replayed with no host launch work.  Inputs are read from, and the result
    written to, the tensors given here: copy new inputs into them before a
    replay.  The call is run `warmup` times on a side stream first (first
    calls set kernel attributes and look up driver entry points, which a
    capture must not see)."""

    def __init__(self, fn, inputs, out, warmup: int = 2):
        self.fn, self.inputs, self.out = fn, list(inputs), out
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(warmup):
                fn(*self.inputs, out=out)
        torch.cuda.current_stream().wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            fn(*self.inputs, out=out)

    def replay(self):
        self.graph.replay()
        return self.out


def reduce_histogram(hist: torch.Tensor, group=None) -> torch.Tensor:
    """Sums an accumulated routing histogram (co-selection or layer-to-layer
    transition counts, int32 [E,E]) over the ranks of a token-sharded job,
    in place, and returns it.

    Both histograms of "Expert Coupling in MoE Pretraining" (Abstract) are
    sums over tokens, so when each rank routes its own tokens the sum over
    ranks is the histogram of the whole job: the one exchange a
    token-sharded layer has, taken once when the statistic is read (placing
    experts by their co-selection wants the job's counts, identical on every
    rank).  With one process, or no process group, the tensor is unchanged."""
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(hist, op=dist.ReduceOp.SUM, group=group)
    return hist
