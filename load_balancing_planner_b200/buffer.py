"""`Buffer`: the MoonEP user API (MoonEP README, "API guide": `Buffer(...)`,
`dispatch`, `combine`, `prefetch_weight`, `reduce_grad`, `destroy`) over the
C ABI, with the R expert-parallel ranks emulated on one GPU.

Argument marshalling only: every call below is one or two calls of the C ABI
(`moonep.py`); the only other device work is the allocation of output tensors.

Emulation.  Every per-rank tensor of the API carries a leading [R]:
hidden [R,S,H], route weights and top-k [R,S,K], local counts [R,E], the
dispatched buffer [R,NvS,H].  Rows [0,E) of the API's per-projection
[E+B,H,H'] weight and gradient tensors are the single shared [E,H,H'] tensor
(on real hardware each rank maps every home rank's rows); rows [E,E+B) of
rank r are `pool[r]` / `reduce_buffer[r]` of an [R,B,H,H'] tensor.

Backward pair (MoonEP README, "dispatch bwd" and "combine bwd"):
  combine backward  = `dispatch(grad_output, plan=plan)`: a scatter with the
                      saved plan, no planning and no weights;
  dispatch backward = `combine(plan, grad_hidden_nvs)`: the unweighted sum of
                      each token's K copies, plus `reduce_grad` for the
                      redundant experts' weight gradients.
The gradient of the route weights travels the same way: scatter it to buffer
order with the plan, or gather a per-slot quantity back to [R,S,K] with
`combine(..., route_weights_nvs=per_slot)`, whose second output is exactly
`per_slot[dst]`.
"""
from __future__ import annotations

import torch

from . import moonep


_STATUS_NAMES = ((moonep.STATUS_BAD_EXPERT, "expert id outside [0, E)"),
                 (moonep.STATUS_DUP_EXPERT, "an expert twice in one token"),
                 (moonep.STATUS_COUNT_MISMATCH, "tokens_per_expert differs from the top-k histogram"),
                 (moonep.STATUS_BAD_PLAN, "inconsistent plan"),
                 (moonep.STATUS_TIMEOUT, "planner barrier timed out"))


class PlanStatusError(RuntimeError):
    """The planner rejected the routing; `status` holds the MOONEP_STATUS_* bits."""

    def __init__(self, status: int):
        why = "; ".join(n for b, n in _STATUS_NAMES if status & b) or "unknown"
        super().__init__(f"plan status {status:#x}: {why}")
        self.status = status


class Buffer:
    """One MoE layer shape: S tokens per rank, hidden size H, top-K routing
    over E experts on `num_ep_ranks` ranks, B prefetch slots per rank.

    `B` defaults to E // num_ep_ranks, the value training requires.
    `num_sms` caps the SMs of the copy kernels; None uses every SM (the
    pages default to 32 because their communication kernels share the GPU
    with expert GEMMs; an emulated layer is a pure HBM copy and wants all).
    `mode` is moonep.TRAINING, moonep.TRAINING_FEWEST_COPIES (a donor gives
    away its largest experts, so recipients hold fewer copies),
    moonep.INFERENCE (overflow home rows; slots to the first B received
    experts) or moonep.INFERENCE_BY_COUNT (slots to the B received experts
    with the most picks).
    """

    def __init__(self, S: int, H: int, K: int, E: int, num_ep_ranks: int, num_sms: int | None = None,
                 token_padding: int = 128, B: int | None = None, mode: int = moonep.TRAINING,
                 device: torch.device | None = None):
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        with torch.cuda.device(self.device):
            self.handle = moonep.moonep_create(S, H, K, E, num_ep_ranks, B, token_padding,
                                               num_sms or 0, mode)
        self.S, self.H, self.K, self.E = S, H, K, E
        self.R = num_ep_ranks
        self.B = self.handle.B
        self.nvs = self.handle.nvs
        self.mode = mode
        self._comm = None
        # the static communication buffer that zero_copy dispatch returns views of
        self._hidden_nvs = None
        self._weights_nvs = None

    # ---- helpers ---------------------------------------------------------
    def _alive(self):
        if self.handle is None:
            raise RuntimeError("Buffer used after destroy()")

    def _run(self, async_finish, inputs, fn):
        """Run fn(stream) on the current stream, or on the communication
        stream after it waits for the current one (async_finish); then the
        result and a CUDA event recorded after the work (or None)."""
        self._alive()
        if not async_finish:
            return fn(torch.cuda.current_stream(self.device)), None
        if self._comm is None:
            self._comm = torch.cuda.Stream(self.device)
        self._comm.wait_stream(torch.cuda.current_stream(self.device))
        for t in inputs:
            if t is not None:
                t.record_stream(self._comm)
        with torch.cuda.stream(self._comm):
            out = fn(self._comm)
        ev = torch.cuda.Event()
        ev.record(self._comm)
        return out, ev

    def _static_nvs(self, weights: bool):
        if self._hidden_nvs is None:
            self._hidden_nvs = torch.empty((self.R, self.nvs, self.H), dtype=torch.bfloat16, device=self.device)
        if weights and self._weights_nvs is None:
            self._weights_nvs = torch.empty((self.R, self.nvs), dtype=torch.float32, device=self.device)
        return self._hidden_nvs, (self._weights_nvs if weights else None)

    # ---- API -------------------------------------------------------------
    def dispatch(self, hidden, route_weights=None, topk_experts=None, tokens_per_expert=None, *,
                 plan: moonep.Plan | None = None, zero_copy: bool = False, async_finish: bool = False):
        """Plan (unless `plan` is given) and scatter.

        Returns (hidden_nvs [R,NvS,H] bf16, route_weights_nvs [R,NvS] fp32 or
        None, cu_seqlens [R,E+B] int32, plan), plus a CUDA event when
        async_finish.  Padding slots of hidden_nvs are not written.  With
        zero_copy the first two are views of the Buffer's static buffer,
        which the next dispatch overwrites."""
        if plan is None and topk_experts is None:
            raise ValueError("dispatch needs topk_experts, or a saved plan")
        h = self.handle

        def go(stream):
            p = plan
            if p is None:
                p = moonep.moonep_plan(h, topk_experts, tokens_per_expert, stream=stream)
            if zero_copy:
                buf, wbuf = self._static_nvs(route_weights is not None)
            else:
                buf, wbuf = None, None
            buf, wbuf = moonep.moonep_dispatch(h, p, hidden, route_weights, buf, wbuf, stream=stream)
            return buf, wbuf, p.cu_seqlens, p

        out, ev = self._run(async_finish, (hidden, route_weights, topk_experts, tokens_per_expert), go)
        return (*out, ev) if async_finish else out

    def combine(self, plan: moonep.Plan, hidden_nvs, route_weights_nvs=None, *, zero_copy: bool = False,
                async_finish: bool = False):
        """out[r,t] = bf16(sum_k w_k * hidden_nvs[dst[r,t,k]]), fp32 sum; w_k = 1
        without route_weights_nvs.  Returns (out [R,S,H] bf16,
        gathered_route_weights [R,S,K] fp32 or None, None), plus a CUDA event
        when async_finish.  zero_copy asserts that the inputs are the views
        the last zero_copy dispatch returned.  On one GPU the input is read
        in place either way: the copy into the communication buffer that the
        pages make without zero_copy is what lets peer ranks read it."""
        if zero_copy:
            if self._hidden_nvs is None or hidden_nvs.data_ptr() != self._hidden_nvs.data_ptr():
                raise ValueError("zero_copy combine takes the hidden_nvs view that dispatch returned")
            if route_weights_nvs is not None and (
                    self._weights_nvs is None or route_weights_nvs.data_ptr() != self._weights_nvs.data_ptr()):
                raise ValueError("zero_copy combine takes the route_weights_nvs view that dispatch returned")
        h = self.handle

        def go(stream):
            o, gw = moonep.moonep_combine(h, plan, hidden_nvs, route_weights_nvs, stream=stream)
            return o, gw, None

        out, ev = self._run(async_finish, (hidden_nvs, route_weights_nvs), go)
        return (*out, ev) if async_finish else out

    def prefetch_weight(self, plan: moonep.Plan, weights, pools, *, async_finish: bool = False):
        """pools[i][r][b] <- weights[i][slot_expert[r][b]] for every used slot:
        `weights` are the [E,H,H'] bf16 projections (gate, up, down, ...),
        `pools` the matching [R,B,H,H'] bf16 slot tensors.  Returns the CUDA
        event when async_finish, else None."""
        weights, pools = list(weights), list(pools)
        _, ev = self._run(async_finish, (*weights, *pools),
                          lambda s: moonep.moonep_prefetch_weight(self.handle, plan, weights, pools, stream=s))
        return ev

    def reduce_grad(self, plan: moonep.Plan, grads, reduce_buffers, *, async_finish: bool = False):
        """grads[i][e] += the slots of reduce_buffers[i] that hold expert e,
        in ascending (rank, slot) order; those slots are then zeroed.
        `grads` are [E,H,H'] fp32, `reduce_buffers` [R,B,H,H'] fp32.  Returns
        the CUDA event when async_finish, else None."""
        grads, reduce_buffers = list(grads), list(reduce_buffers)
        _, ev = self._run(async_finish, (*grads, *reduce_buffers),
                          lambda s: moonep.moonep_reduce_grad(self.handle, plan, grads, reduce_buffers, stream=s))
        return ev

    def check(self, plan: moonep.Plan) -> None:
        """Raise if the planner flagged the routing (reads the device status
        word; the one call here that waits for the device)."""
        st = moonep.moonep_read_status(plan)
        if st:
            raise PlanStatusError(st)

    def destroy(self) -> None:
        """Release the handle and the static buffers."""
        if self._comm is not None:
            self._comm.synchronize()
        self._hidden_nvs = self._weights_nvs = None
        if self.handle is not None:
            self.handle.close()
            self.handle = None
