"""Seeded synthetic inputs shaped like the router workloads of the pages' model
families.  Only input generation lives here: no routing arithmetic.

Workloads (shapes and distributions; "I modelli MoE open hanno router opposti"
gives the expert counts, k, scoring and shared experts of the families;
"DeepSeek-V3.2-Exp - Select experts" the 8 x 32 groups, keep 4, top 8):
  mixtral_tiny   T=256, E=8, k=2, softmax, renormalised; logits ~N(0,1) given;
                 x, expert outputs bf16 d=128 ~N(0,1)
  qwen3_dynk     T=16384, d=2048, E=128, softmax, renormalised, no shared; gate
                 x ~N(0,1), W ~N(0,0.02^2) bf16; k drawn from {4,8,16} per
                 contiguous 512-token request segment (k_max = 16)
  deepseek_v3    T=65536, d=7168, E=256, k=8, sigmoid; selection bias ~U(-0.1,0.1)
                 fp32; 8 groups of 32, group score = sum of top 2, keep 4;
                 renormalised, route_scale 2.5; one shared expert in combine
  deepseek_v4    T=65536, d=7168, E=384, k=6, sqrt-softplus, renormalised; the
                 path ends at permute; hash layer: token ids ~U[0,129280),
                 tid2eid [129280][6] ~U[0,384)
  llama4_top1    T=262144, d=5120, E=128, k=1, sigmoid without renormalisation,
                 one shared expert; logits ~N(0,1), 10% of rows +3 on 4 hot experts
  gptoss_top4    T=262144, d=2880, E=128, k=4, gpt-oss (softmax over the 4
                 selected logits); logits as llama4_top1
  with_ffn()      mixtral_tiny, qwen3_dynk and gptoss_top4 also run their experts'
                 SwiGLU FFN (F = 256, 768, 2880; gpt-oss: clamped SwiGLU with
                 biases) on the permuted rows, with synthetic weights
  llama4_top1_capacity
                 llama4_top1 with a Switch-style capacity (factor 1.0: each
                 expert keeps at most T/E = 2048 tokens, the skewed hot experts
                 drop the rest) and expert blocks padded to 128 rows
Seeds: 1000 * workload index + tensor index.  bf16 tensors are drawn in fp32
and rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    T: int
    d: int
    E: int
    k_max: int
    score: str
    gate: bool                    # logits come from the gate GEMM (else given ~N(0,1))
    bias: bool = False
    n_groups: int = 1
    topk_groups: int = 1
    group_topn: int = 1
    renormalize: bool = True
    route_scale: float = 1.0
    shared: bool = False
    k_choices: tuple | None = None  # per-request k, one draw per segment
    segment: int = 512
    skew: bool = False
    combine: bool = True           # the path ends at combine (else at permute)
    hash_vocab: int = 0            # > 0: a hash-routed layer is part of the workload
    w_std: float = 0.02
    capacity_factor: float = 0.0   # > 0: per-expert capacity ceil(cf * T * k / E)
    pad: int = 1                   # expert blocks padded to a multiple of this many rows
    ffn_dim: int = 0               # expert FFN width F (0: no FFN model for this family)
    ffn_act: str = "swiglu"        # "swiglu" or "swiglu_oai" (gpt-oss, with biases)

    @property
    def limited(self) -> bool:
        """Dispatch with a capacity and/or padded expert blocks."""
        return self.capacity_factor > 0 or self.pad > 1

    @property
    def capacity(self) -> int:
        if self.capacity_factor <= 0:
            return 0
        return max(1, math.ceil(self.capacity_factor * self.T * self.k_max / self.E))

    def scaled(self, T: int) -> "Workload":
        """Same workload with another token count (smaller parity cases)."""
        return dataclasses.replace(self, T=T)

    def with_ffn(self) -> "Workload":
        """The workload with its experts' FFN run on the permuted rows: expert
        blocks padded to the 128-row tiles of the grouped GEMMs."""
        if not self.ffn_dim:
            raise ValueError(f"{self.name} has no expert FFN shape")
        return dataclasses.replace(self, pad=max(self.pad, 128))


WORKLOADS = {
    w.name: w for w in [
        Workload("mixtral_tiny", 1, T=256, d=128, E=8, k_max=2, score="softmax", gate=False,
                 ffn_dim=256),
        Workload("qwen3_dynk", 2, T=16384, d=2048, E=128, k_max=16, score="softmax", gate=True,
                 k_choices=(4, 8, 16), ffn_dim=768),
        Workload("deepseek_v3", 3, T=65536, d=7168, E=256, k_max=8, score="sigmoid", gate=True,
                 bias=True, n_groups=8, topk_groups=4, group_topn=2, route_scale=2.5,
                 shared=True),
        Workload("deepseek_v4", 4, T=65536, d=7168, E=384, k_max=6, score="sqrt_softplus",
                 gate=True, combine=False, hash_vocab=129280),
        Workload("llama4_top1", 5, T=262144, d=5120, E=128, k_max=1, score="sigmoid",
                 gate=False, renormalize=False, shared=True, skew=True),
        Workload("gptoss_top4", 6, T=262144, d=2880, E=128, k_max=4, score="topk_softmax",
                 gate=False, skew=True, ffn_dim=2880, ffn_act="swiglu_oai"),
        Workload("llama4_top1_capacity", 7, T=262144, d=5120, E=128, k_max=1, score="sigmoid",
                 gate=False, renormalize=False, shared=True, skew=True, capacity_factor=1.0,
                 pad=128),
    ]
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_bf16(shape, std, device, seed):
    t = torch.randn(shape, generator=_gen(device, seed), device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def make_expert_weights(wl: Workload, device="cuda", seed_offset: int = 0) -> dict:
    """Synthetic expert FFN weights: W1, W3 [E][F][d] ~N(0, 1/d), W2 [E][d][F]
    ~N(0, 1/F) in bf16 (so the projections are O(1) for O(1) inputs); for the
    gpt-oss activation also biases b1, b3 [E][F] and b2 [E][d] ~N(0, 0.5^2)."""
    s = 1000 * wl.index + 20 + seed_offset
    E, d, F = wl.E, wl.d, wl.ffn_dim
    out = {"w1": normal_bf16((E, F, d), d ** -0.5, device, s),
           "w3": normal_bf16((E, F, d), d ** -0.5, device, s + 1),
           "w2": normal_bf16((E, d, F), F ** -0.5, device, s + 2),
           "b1": None, "b3": None, "b2": None}
    if wl.ffn_act == "swiglu_oai":
        for i, (name, shape) in enumerate((("b1", (E, F)), ("b3", (E, F)), ("b2", (E, d)))):
            out[name] = torch.randn(shape, generator=_gen(device, s + 3 + i), device=device) * 0.5
    return out


def k_per_token(wl: Workload, device, seed=None):
    """k_t for every token: one draw from wl.k_choices per request segment."""
    if wl.k_choices is None:
        return None
    seed = 1000 * wl.index + 3 if seed is None else seed
    nseg = math.ceil(wl.T / wl.segment)
    choices = torch.tensor(wl.k_choices, dtype=torch.int32, device=device)
    pick = torch.randint(0, len(wl.k_choices), (nseg,), generator=_gen(device, seed),
                         device=device)
    return choices[pick].repeat_interleave(wl.segment)[: wl.T].contiguous()


def num_assignments(wl: Workload, kpt) -> int:
    """N = total routing slots that will be filled (sum of per-token k)."""
    return int(kpt.sum().item()) if kpt is not None else wl.T * wl.k_max


def expert_rows(wl: Workload, kpt) -> int:
    """Rows of the expert-ordered buffers (xs, y): N, or with a capacity and
    padded blocks the most they can need, min(N, E * capacity) + E * (pad - 1)."""
    n = num_assignments(wl, kpt)
    if not wl.limited:
        return n
    if wl.capacity:
        n = min(n, wl.E * wl.capacity)
    return n + wl.E * (wl.pad - 1)


def make_inputs(wl: Workload, device="cuda", *, with_y=True, with_x=True,
                seed_offset: int = 0) -> dict:
    """All seeded inputs of one workload on ``device``.

    Keys: x [T,d] bf16, w [E,d] bf16 (gate workloads) or logits [T,E] fp32,
    bias [E] fp32, k_per_token [T] int32, y [N,d] bf16 (synthetic expert
    outputs in expert-contiguous order), shared [T,d] bf16, token_ids [T] and
    tid2eid [vocab,k] int32 (hash layer).  Absent pieces are None.
    """
    s = 1000 * wl.index + seed_offset
    out = {k: None for k in ("x", "w", "logits", "bias", "k_per_token", "y", "shared",
                             "token_ids", "tid2eid")}
    if with_x:
        out["x"] = normal_bf16((wl.T, wl.d), 1.0, device, s + 0)
    if wl.gate:
        out["w"] = normal_bf16((wl.E, wl.d), wl.w_std, device, s + 1)
    else:
        lg = torch.randn((wl.T, wl.E), generator=_gen(device, s + 1), device=device)
        if wl.skew:
            n_hot_rows = round(0.1 * wl.T)
            rows = torch.randperm(wl.T, generator=_gen(device, s + 5), device=device)[:n_hot_rows]
            hot = torch.randperm(wl.E, generator=_gen(device, s + 6), device=device)[:4]
            lg[rows.unsqueeze(1), hot.unsqueeze(0)] += 3.0
        out["logits"] = lg.contiguous()
    if wl.bias:
        b = torch.rand((wl.E,), generator=_gen(device, s + 2), device=device)
        out["bias"] = (b * 0.2 - 0.1).contiguous()
    out["k_per_token"] = k_per_token(wl, device, s + 3)
    if with_y and wl.combine:
        n = expert_rows(wl, out["k_per_token"])
        out["y"] = normal_bf16((n, wl.d), 1.0, device, s + 4)
    if wl.shared and wl.combine:
        out["shared"] = normal_bf16((wl.T, wl.d), 1.0, device, s + 7)
    if wl.hash_vocab:
        out["token_ids"] = torch.randint(0, wl.hash_vocab, (wl.T,), generator=_gen(device, s + 8),
                                         device=device, dtype=torch.int32)
        out["tid2eid"] = torch.randint(0, wl.E, (wl.hash_vocab, wl.k_max),
                                       generator=_gen(device, s + 9), device=device,
                                       dtype=torch.int32)
    return out
