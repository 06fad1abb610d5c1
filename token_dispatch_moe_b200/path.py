"""The router-and-dispatch chain as one object: buffers plus the C-ABI calls in
order (gate -> route -> dispatch -> permute -> combine), all on one stream.

Only orchestration lives here: torch allocates device memory, and every step
is a call into libmoe_dispatch.so.  The expert FFN between permute and combine
is outside the path; its outputs ``y`` are an input of :meth:`RouterDispatch.run`.
"""
from __future__ import annotations

import torch

from . import (MOE_ACT_SWIGLU, MOE_ACT_SWIGLU_OAI, RouteParams, moe_combine, moe_dispatch,
               moe_dispatch_limited, moe_dispatch_limited_rows, moe_dispatch_workspace_size,
               moe_expert_down, moe_expert_gate_up, moe_gate_gemm, moe_gate_route,
               moe_hash_route, moe_permute, moe_route)
from .workloads import Workload


class RouterDispatch:
    """Preallocated buffers for T tokens of one layer configuration."""

    def __init__(self, wl: Workload, device="cuda", n_rows: int | None = None,
                 fused: bool | None = None, keep_logits: bool = False):
        """fused: gate workloads route inside the gate GEMM (moe_gate_route)
        when the configuration allows it (k_max <= 16); None picks it where it
        measured faster: a gate workload with neither a group limit nor a
        per-token k.  (The epilogue routes on the GEMM's four epilogue warps
        only: a group limit's extra passes, or a selection network sized for
        k_max = 16 when most tokens take 4 or 8, cost more there than the
        separate route kernel spread over the whole GPU.)
        keep_logits: also write the logits (parity checks need them; the fused
        path skips them otherwise)."""
        self.wl = wl
        if fused is None:
            fused = wl.n_groups == 1 and wl.k_choices is None
        self.fused = bool(fused and wl.gate and wl.k_max <= 16)
        self.keep_logits = keep_logits or not self.fused
        self.params = RouteParams.make(wl.E, wl.k_max, wl.score, wl.n_groups, wl.topk_groups,
                                       wl.group_topn, wl.renormalize, wl.route_scale)
        T, E, k = wl.T, wl.E, wl.k_max
        i32 = dict(dtype=torch.int32, device=device)
        self.logits = (torch.empty((T, E), dtype=torch.float32, device=device)
                       if wl.gate and self.keep_logits else None)
        self.topk_ids = torch.empty((T, k), **i32)
        self.topk_w = torch.empty((T, k), dtype=torch.float32, device=device)
        self.counts = torch.empty((E,), **i32)
        self.offsets = torch.empty((E + 1,), **i32)
        # With a capacity or padded expert blocks (moe_dispatch_limited) the
        # expert-ordered buffers hold the bound that call states.
        self.capacity = wl.capacity if wl.limited else 0
        self.expert_rows = (moe_dispatch_limited_rows(T, k, E, self.capacity, wl.pad)
                            if wl.limited else T * k)
        self.sorted_token = torch.empty((max(self.expert_rows, 1),), **i32)
        self.dest_pos = torch.empty((T, k), **i32)
        self.dropped = torch.zeros((1,), **i32) if wl.limited else None
        ws = moe_dispatch_workspace_size(T, k, E)
        self.workspace = torch.empty((max(ws, 256),), dtype=torch.uint8, device=device)
        rows = self.expert_rows if n_rows is None else n_rows
        self.xs = torch.empty((max(rows, 1), wl.d), dtype=torch.bfloat16, device=device)
        self.out = (torch.empty((T, wl.d), dtype=torch.bfloat16, device=device)
                    if wl.combine else None)
        self.status = torch.zeros((1,), **i32)
        self.h = self.y = None
        if wl.ffn_dim and wl.pad % 128 == 0:  # the experts' FFN can run on these blocks
            self.h = torch.empty((max(self.expert_rows, 1), wl.ffn_dim), dtype=torch.bfloat16,
                                 device=device)
            self.y = torch.empty((max(self.expert_rows, 1), wl.d), dtype=torch.bfloat16,
                                 device=device)
        if wl.hash_vocab:
            self.hash_ids = torch.empty((T, k), **i32)
            self.hash_w = torch.empty((T, k), dtype=torch.float32, device=device)

    # Individual steps (each one C-ABI call) -----------------------------------
    def gate(self, x, w, stream=None):
        moe_gate_gemm(x, w, self.logits, self.status, stream)
        return self.logits

    def gate_route(self, x, w, bias=None, k_per_token=None, stream=None):
        moe_gate_route(x, w, bias, k_per_token, self.params, self.topk_ids, self.topk_w,
                       self.logits, self.status, stream)

    def route(self, logits, bias=None, k_per_token=None, stream=None):
        moe_route(logits, bias, k_per_token, self.params, self.topk_ids, self.topk_w,
                  self.status, stream)

    def hash_route(self, token_ids, tid2eid, logits=None, stream=None):
        moe_hash_route(token_ids, tid2eid, logits, self.params, self.hash_ids, self.hash_w,
                       self.status, stream)

    def dispatch(self, ids=None, stream=None):
        ids = self.topk_ids if ids is None else ids
        if self.wl.limited:
            moe_dispatch_limited(ids, self.wl.E, self.capacity, self.wl.pad, self.counts,
                                 self.offsets, self.sorted_token, self.dest_pos, self.workspace,
                                 self.dropped, self.status, stream)
        else:
            moe_dispatch(ids, self.wl.E, self.counts, self.offsets, self.sorted_token,
                         self.dest_pos, self.workspace, self.status, stream)

    def permute(self, x, stream=None):
        moe_permute(x, self.dest_pos, self.xs, stream)

    def combine(self, y, shared=None, stream=None):
        moe_combine(y, self.topk_w, self.dest_pos, shared, self.out, stream)

    def expert_gate_up(self, weights: dict, stream=None):
        act = MOE_ACT_SWIGLU_OAI if self.wl.ffn_act == "swiglu_oai" else MOE_ACT_SWIGLU
        moe_expert_gate_up(self.xs, self.offsets, weights["w1"], weights["w3"], self.h,
                           weights["b1"], weights["b3"], act, self.status, stream)

    def expert_down(self, weights: dict, stream=None):
        moe_expert_down(self.h, self.offsets, weights["w2"], self.y, weights["b2"], self.status,
                        stream)

    # The whole chain -----------------------------------------------------------
    def run(self, inputs: dict, stream=None, experts: dict | None = None):
        """gate (if the workload has one) -> route -> dispatch -> permute ->
        [experts' FFN, when ``experts`` holds their weights] -> combine (if the
        workload ends there).  ``inputs`` as made by :func:`workloads.make_inputs`;
        without experts the combine reads the synthetic ``inputs["y"]``."""
        if self.fused:
            self.gate_route(inputs["x"], inputs["w"], inputs["bias"], inputs["k_per_token"], stream)
        else:
            logits = (self.gate(inputs["x"], inputs["w"], stream) if self.wl.gate
                      else inputs["logits"])
            self.route(logits, inputs["bias"], inputs["k_per_token"], stream)
        self.dispatch(stream=stream)
        self.permute(inputs["x"], stream)
        y = inputs["y"]
        if experts is not None:
            self.expert_gate_up(experts, stream)
            self.expert_down(experts, stream)
            y = self.y
        if self.wl.combine:
            self.combine(y, inputs["shared"], stream)
        return self.out if self.wl.combine else self.xs

    def run_hash_layer(self, inputs: dict, logits=None, stream=None):
        """hash_route -> dispatch -> permute (the hash-routed layer's chain)."""
        self.hash_route(inputs["token_ids"], inputs["tid2eid"], logits, stream)
        self.dispatch(self.hash_ids, stream)
        self.permute(inputs["x"], stream)
        return self.xs
