"""Seeded synthetic inputs for the linear-attention workloads.

This module is shared by the tests, the benchmark and the smoke check.  It holds the
input recipes only -- shapes, distributions, seeds and draw order -- and none of the
method's arithmetic.  Both the fp64 oracle and the CUDA library receive the tensors it
returns (the oracle after an exact upcast to fp64).

Draw order is fixed: q, k, v, gate pre-activation x, beta pre-activation y (and, for
decode, the initial state first).  Gates are stored as values a_t in (0, 1], not logs;
in mode 3 (Kimi Delta Attention) there is one gate per channel, x of shape [.., d_k].
"""
from __future__ import annotations

import dataclasses
import math

import torch

MODE_ELU1_NORM = 0
MODE_GATED = 1
MODE_GATED_DELTA = 2
MODE_KDA = 3
MODE_RETNET = 4


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    mode: int
    dtype: torch.dtype          # q, k, v, o; state, z, gate and beta are always fp32
    B: int                      # batch (prefill) or sequences N (decode)
    H: int
    T: int                      # tokens per sequence (prefill) or decode steps
    dk: int
    dv: int
    seed: int
    chunk: int = 0              # 0 -> the library default
    qk_scale: float = 1.0       # q, k ~ N(0,1) * qk_scale
    v_scale: float = 1.0
    qk_l2norm: bool = False     # L2-normalise q, k rows in fp32 before the cast
    gate: str = "none"          # "none" | "softplus" (a = exp(-softplus(x + gate_shift))) |
                                # "retnet" (mode 4: one constant gate per head, no draw)
    gate_shift: float = 0.0
    beta: bool = False          # beta = sigmoid(y), y ~ N(0,1)
    decode: bool = False
    state_std: float = 0.0      # decode: initial state ~ N(0, state_std^2)

    @property
    def tokens(self) -> int:
        """Tokens processed per step: B*T for prefill, N for one decode step."""
        return self.B if self.decode else self.B * self.T


# The five workloads, restated from the task's configuration list.
CONFIGS = {
    "elu1_f32_small": Workload("elu1_f32_small", MODE_ELU1_NORM, torch.float32, B=1, H=2, T=256,
                               dk=64, dv=64, seed=1),
    "elu1_bf16_b4h16t4096": Workload("elu1_bf16_b4h16t4096", MODE_ELU1_NORM, torch.bfloat16, B=4,
                                     H=16, T=4096, dk=128, dv=128, seed=2, chunk=64,
                                     qk_scale=1 / math.sqrt(128), v_scale=1 / math.sqrt(128)),
    "gated_bf16_b8h16t8192": Workload("gated_bf16_b8h16t8192", MODE_GATED, torch.bfloat16, B=8,
                                      H=16, T=8192, dk=128, dv=128, seed=3,
                                      qk_scale=1 / math.sqrt(128), gate="softplus"),
    "gdn_bf16_b2h16t32768": Workload("gdn_bf16_b2h16t32768", MODE_GATED_DELTA, torch.bfloat16,
                                     B=2, H=16, T=32768, dk=128, dv=128, seed=4, qk_l2norm=True,
                                     gate="softplus", beta=True),
    "gdn_decode_n256h32": Workload("gdn_decode_n256h32", MODE_GATED_DELTA, torch.bfloat16, B=256,
                                   H=32, T=1000, dk=128, dv=128, seed=5, qk_l2norm=True,
                                   gate="softplus", beta=True, decode=True, state_std=0.02),
    # Kimi Delta Attention (per-channel gates): the shapes and recipes of the two
    # gated-delta workloads above with a_t drawn per channel.
    "kda_bf16_b2h16t32768": Workload("kda_bf16_b2h16t32768", MODE_KDA, torch.bfloat16, B=2, H=16,
                                     T=32768, dk=128, dv=128, seed=6, qk_l2norm=True,
                                     gate="softplus", beta=True),
    "kda_decode_n256h32": Workload("kda_decode_n256h32", MODE_KDA, torch.bfloat16, B=256, H=32,
                                   T=1000, dk=128, dv=128, seed=7, qk_l2norm=True,
                                   gate="softplus", beta=True, decode=True, state_std=0.02),
    # Constant per-head decay (RetNet / Lightning attention) on the scalar-gated shapes.
    "retnet_bf16_b8h16t8192": Workload("retnet_bf16_b8h16t8192", MODE_RETNET, torch.bfloat16, B=8,
                                       H=16, T=8192, dk=128, dv=128, seed=10,
                                       qk_scale=1 / math.sqrt(128), gate="retnet"),
    # Profiling cases of the gated delta rule and KDA (counter captures need a few GB on the
    # device at most): the B2 H16 recipe at a quarter of its length (200 MB of inputs, more than
    # L2), and 8 heads, which take the segmented kernels.
    "gdn_bf16_b2h16t8192": Workload("gdn_bf16_b2h16t8192", MODE_GATED_DELTA, torch.bfloat16, B=2,
                                    H=16, T=8192, dk=128, dv=128, seed=4, qk_l2norm=True,
                                    gate="softplus", beta=True),
    "gdn_bf16_b1h8t16384": Workload("gdn_bf16_b1h8t16384", MODE_GATED_DELTA, torch.bfloat16, B=1,
                                    H=8, T=16384, dk=128, dv=128, seed=4, qk_l2norm=True,
                                    gate="softplus", beta=True),
    # the KDA recipe at a quarter of its length (600 MB of inputs with the per-channel gates)
    "kda_bf16_b2h16t8192": Workload("kda_bf16_b2h16t8192", MODE_KDA, torch.bfloat16, B=2, H=16,
                                    T=8192, dk=128, dv=128, seed=6, qk_l2norm=True,
                                    gate="softplus", beta=True),
}


def _qkv(w: Workload, gen: torch.Generator, device, lead):
    """Draw q, k, v (in that order) with leading shape `lead`."""
    q = torch.randn(*lead, w.dk, generator=gen, device=device, dtype=torch.float32)
    k = torch.randn(*lead, w.dk, generator=gen, device=device, dtype=torch.float32)
    v = torch.randn(*lead, w.dv, generator=gen, device=device, dtype=torch.float32)
    if w.qk_l2norm:
        q = q / q.norm(dim=-1, keepdim=True)
        k = k / k.norm(dim=-1, keepdim=True)
    else:
        q = q * w.qk_scale
        k = k * w.qk_scale
    v = v * w.v_scale
    return q.to(w.dtype), k.to(w.dtype), v.to(w.dtype)


def _gates(w: Workload, gen: torch.Generator, device, lead):
    gate = beta = None
    if w.gate == "retnet":
        # RetNet's per-head decays: gamma_h = 1 - 2^(-5 - 8 h / H), from 0.969 towards 1
        h = torch.arange(w.H, device=device, dtype=torch.float64)
        gate = (1.0 - torch.pow(2.0, -5.0 - 8.0 * h / w.H)).to(torch.float32)
    elif w.gate == "softplus":
        shape = (*lead, w.dk) if w.mode == MODE_KDA else lead
        x = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
        # a = exp(-softplus(x)) = sigmoid(-x): a value in (0, 1)
        gate = torch.exp(-torch.nn.functional.softplus(x + w.gate_shift))
    elif w.gate != "none":
        raise ValueError(f"unknown gate recipe {w.gate!r}")
    if w.beta:
        y = torch.randn(*lead, generator=gen, device=device, dtype=torch.float32)
        beta = torch.sigmoid(y)
    return gate, beta


def prefill_inputs(w: Workload, device="cpu", init_state_std: float = 0.0):
    """q,k [B,H,T,d_k], v [B,H,T,d_v] in w.dtype; gate, beta [B,H,T] fp32 or None (mode 3:
    gate [B,H,T,d_k]);
    state0 [B,H,d_v,d_k] fp32 (zeros unless init_state_std > 0)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    lead = (w.B, w.H, w.T)
    q, k, v = _qkv(w, gen, device, lead)
    gate, beta = _gates(w, gen, device, lead)
    if init_state_std > 0:
        state0 = torch.randn(w.B, w.H, w.dv, w.dk, generator=gen, device=device) * init_state_std
    else:
        state0 = torch.zeros(w.B, w.H, w.dv, w.dk, device=device)
    return dict(q=q, k=k, v=v, gate=gate, beta=beta, state0=state0)


def decode_inputs(w: Workload, steps: int | None = None, device="cpu", n_seqs: int | None = None):
    """Initial state [N,H,d_v,d_k] ~ N(0, state_std^2) and per-step inputs stacked over
    steps: q,k [steps,N,H,d_k], v [steps,N,H,d_v], gate, beta [steps,N,H] (mode 3: gate
    [steps,N,H,d_k])."""
    steps = w.T if steps is None else steps
    N = w.B if n_seqs is None else n_seqs
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    state0 = torch.randn(N, w.H, w.dv, w.dk, generator=gen, device=device) * w.state_std
    lead = (steps, N, w.H)
    q, k, v = _qkv(w, gen, device, lead)
    gate, beta = _gates(w, gen, device, lead)
    z0 = None
    if w.mode == MODE_ELU1_NORM:
        z0 = torch.rand(N, w.H, w.dk, generator=gen, device=device) + 1.0
    return dict(state0=state0, z0=z0, q=q, k=k, v=v, gate=gate, beta=beta)


def variant(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields changed (smaller sizes, weaker decay ...)."""
    return dataclasses.replace(w, **changes)


# The backward pass of the scalar-gated prefill (mode 1): the default prefill's shape
# (B4 H16 T4096, d = 128, bf16) with the gated recipe; output cotangents dO ~ N(0, 1).
# The delta rule's backward (mode 2) on the long-context Gated DeltaNet prefill's shape and
# recipe (B2 H16 T32768, d = 128, bf16, L2-normalised q and k, b = sigmoid(N(0, 1))).
BACKWARD_CONFIGS = {
    "gated_bwd_bf16_b4h16t4096": Workload("gated_bwd_bf16_b4h16t4096", MODE_GATED, torch.bfloat16,
                                          B=4, H=16, T=4096, dk=128, dv=128, seed=11,
                                          qk_scale=1 / math.sqrt(128), gate="softplus"),
    "gdn_bwd_bf16_b2h16t32768": Workload("gdn_bwd_bf16_b2h16t32768", MODE_GATED_DELTA, torch.bfloat16,
                                         B=2, H=16, T=32768, dk=128, dv=128, seed=12,
                                         qk_l2norm=True, gate="softplus", gate_shift=-3.0, beta=True),
    # profiling case: the same recipe at an eighth of the length (counter captures)
    "gdn_bwd_bf16_b2h16t4096": Workload("gdn_bwd_bf16_b2h16t4096", MODE_GATED_DELTA, torch.bfloat16,
                                        B=2, H=16, T=4096, dk=128, dv=128, seed=12,
                                        qk_l2norm=True, gate="softplus", gate_shift=-3.0, beta=True),
}


# ---- the short causal convolution in front of q, k, v
@dataclasses.dataclass(frozen=True)
class ConvWorkload:
    name: str
    dtype: torch.dtype          # x, y and the carried window
    B: int
    T: int
    H: int
    dk: int
    dv: int
    width: int
    seed: int
    silu: bool = True           # SiLU on q, k, v
    l2norm_qk: bool = True      # per-head L2 norm of q and k

    @property
    def tokens(self) -> int:
        return self.B * self.T


# The Gated DeltaNet prefill workload's q, k, v (B2 H16 T32768, d = 128) through the
# width-4 convolution of the page, with SiLU and the q/k L2 norm.
CONV_CONFIGS = {
    "conv_bf16_b2h16t32768": ConvWorkload("conv_bf16_b2h16t32768", torch.bfloat16, B=2, T=32768,
                                          H=16, dk=128, dv=128, width=4, seed=8),
}


# A Gated DeltaNet layer's attention path from its projections: the convolution above, then
# the gated-delta prefill workload (its gate and beta recipe), fused in one call
# (la_prefill_conv) or as the separate calls (three la_short_conv, la_prefill).
@dataclasses.dataclass(frozen=True)
class LayerWorkload:
    name: str
    conv: "ConvWorkload"
    prefill: "Workload"
    fused: bool

    @property
    def tokens(self) -> int:
        return self.conv.B * self.conv.T


LAYER_CONFIGS = {
    n: LayerWorkload(n, CONV_CONFIGS["conv_bf16_b2h16t32768"], CONFIGS["gdn_bf16_b2h16t32768"], fused)
    for n, fused in (("gdn_layer_fused_bf16_b2h16t32768", True), ("gdn_layer_split_bf16_b2h16t32768", False))
}


def conv_inputs(B, T, C, width, dtype, seed, device="cpu", window=True):
    """Projection output x [B,T,C] ~ N(0,1), taps w [C,width] ~ N(0,1)/sqrt(width) (fp32),
    carried window [B,width-1,C] ~ N(0,1) (or None).  Draw order: x, w, window."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = torch.randn(B, T, C, generator=gen, device=device, dtype=torch.float32).to(dtype)
    w = torch.randn(C, width, generator=gen, device=device, dtype=torch.float32) / math.sqrt(width)
    win = None
    if window:
        win = torch.randn(B, width - 1, C, generator=gen, device=device,
                          dtype=torch.float32).to(dtype)
    return x, w, win


# ---- packed variable-length sequences
@dataclasses.dataclass(frozen=True)
class VarlenWorkload:
    name: str
    base: Workload              # mode, dtype, H, d, recipes; its B and T are unused
    N: int                      # sequences
    min_len: int
    max_len: int                # lengths log-uniform in [min_len, max_len]

    def lengths(self) -> list:
        return varlen_lengths(self.N, self.min_len, self.max_len, self.base.seed)

    @property
    def tokens(self) -> int:
        return sum(self.lengths())


def varlen_lengths(N, lo, hi, seed):
    """N sequence lengths, log-uniform in [lo, hi] (a serving batch's mix of short and
    long prompts), drawn from their own generator."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed + 777)
    u = torch.rand(N, generator=gen, dtype=torch.float64)
    return [int(round(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo))))) for x in u]


def varlen_inputs(w: Workload, lengths, device="cpu", init_state_std: float = 0.0):
    """Packed q,k [H,T,d_k], v [H,T,d_v], gate/beta [H,T] (mode 3: gate [H,T,d_k]),
    cu_seqlens int32 [N+1] and start states [N,H,d_v,d_k] (zeros unless init_state_std),
    drawn with the recipes of `w` (its B and T are ignored)."""
    T = int(sum(lengths))
    wp = dataclasses.replace(w, B=1, T=T)
    d = prefill_inputs(wp, device=device)
    out = {k: (None if d[k] is None else d[k][0].contiguous()) for k in ("q", "k", "v", "gate", "beta")}
    if w.gate == "retnet":
        out["gate"] = d["gate"]   # one constant per head, [H]: nothing to unpack
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    out["cu"] = torch.tensor(cu, dtype=torch.int32, device=device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed + 4242)
    N = len(lengths)
    if init_state_std > 0:
        out["state0"] = torch.randn(N, w.H, w.dv, w.dk, generator=gen, device=device) * init_state_std
    else:
        out["state0"] = torch.zeros(N, w.H, w.dv, w.dk, device=device)
    return out


# A serving-style batch for the Gated DeltaNet recipe: 64 sequences of 64 .. 8192 tokens.
VARLEN_CONFIGS = {
    "gdn_varlen_bf16_n64h16": VarlenWorkload(
        "gdn_varlen_bf16_n64h16",
        Workload("gdn_varlen_bf16_n64h16", MODE_GATED_DELTA, torch.bfloat16, B=1, H=16, T=0, dk=128,
                 dv=128, seed=9, qk_l2norm=True, gate="softplus", beta=True),
        N=64, min_len=64, max_len=8192),
}
