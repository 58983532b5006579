"""Seeded synthetic workloads shared by the tests, the smoke check and the bench.

This module only draws random inputs; it holds none of the gated delta rule's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Recipe (one CPU ``torch.Generator`` per workload, drawn in the order
q, k, v, g, beta, h0):

  q, k  ~ N(0, 1) in fp32, L2-normalised over the head dimension, then cast to
        the workload dtype (so bf16 keys are normalised up to bf16 rounding; the
        library and the oracle see the same stored values)
  v     ~ N(0, 1), cast to the workload dtype
  g     = logsigmoid(N(mu, 1)) in fp32: [B,T,Hv] for a scalar per-head gate,
        [B,T,Hv,Dk] for a per-key-channel gate
  beta  = sigmoid(N(0, 1)) in fp32, [B,T,Hv]
  h0    = 0.02 * N(0, 1) in fp32, [B,Hv,Dk,Dv] (or absent, meaning zeros)

The shapes and distributions are the five workloads of the gated delta-rule
study: a tiny fp32 GDN case, a nanochat-scale GDN layer, a grouped-value GDN
layer (16 key heads shared by 48 value heads, as in the Qwen GDN blocks of the
Frontier-model atlas, item 08), a KDA layer with a per-channel gate, and a
batch-256 decode loop; plus the layer around the recurrence (make_layer_inputs)
and the backward of the nanochat-scale layer (make_upstream).
"""
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int              # tokens per sequence (chunked forward) or decode steps
    Hk: int
    Hv: int
    Dk: int
    Dv: int
    gate: str           # "scalar" (GDN) or "channel" (KDA)
    dtype: str          # dtype of q, k, v, o: "bf16" or "fp32"
    g_mu: float         # g = logsigmoid(N(g_mu, 1))
    h0_std: float       # 0.0 means h0 absent (zeros)
    seed: int
    decode: bool = False
    layer: bool = False   # inputs are the raw q/k/v projections of the layer (make_layer_inputs)
    bwd: bool = False     # one step is the backward (gdr_bwd) with upstream gradients (make_upstream)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def gate_mode(self) -> int:
        return 0 if self.gate == "scalar" else 1

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def head_tokens(self) -> int:
        return self.B * self.T * self.Hv


WORKLOADS = {
    "tiny_gdn_fp32": Workload("tiny_gdn_fp32", B=1, T=256, Hk=2, Hv=2, Dk=64, Dv=64,
                              gate="scalar", dtype="fp32", g_mu=3.0, h0_std=0.0, seed=0),
    "gdn_bf16": Workload("gdn_bf16", B=8, T=2048, Hk=16, Hv=16, Dk=128, Dv=128,
                         gate="scalar", dtype="bf16", g_mu=3.0, h0_std=0.02, seed=1),
    "gva_gdn_bf16": Workload("gva_gdn_bf16", B=4, T=4096, Hk=16, Hv=48, Dk=128, Dv=128,
                             gate="scalar", dtype="bf16", g_mu=3.0, h0_std=0.02, seed=2),
    "kda_bf16": Workload("kda_bf16", B=2, T=16384, Hk=32, Hv=32, Dk=128, Dv=128,
                         gate="channel", dtype="bf16", g_mu=4.0, h0_std=0.02, seed=3),
    "decode_bf16": Workload("decode_bf16", B=256, T=512, Hk=16, Hv=48, Dk=128, Dv=128,
                            gate="scalar", dtype="bf16", g_mu=3.0, h0_std=0.02, seed=4,
                            decode=True),
    "gdn_layer_bf16": Workload("gdn_layer_bf16", B=8, T=2048, Hk=16, Hv=16, Dk=128, Dv=128,
                               gate="scalar", dtype="bf16", g_mu=3.0, h0_std=0.02, seed=5,
                               layer=True),
    "gdn_bwd_bf16": Workload("gdn_bwd_bf16", B=8, T=2048, Hk=16, Hv=16, Dk=128, Dv=128,
                             gate="scalar", dtype="bf16", g_mu=3.0, h0_std=0.02, seed=6, bwd=True),
}


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_inputs(w: Workload, device="cpu"):
    """Draw the workload's inputs on the CPU (deterministic), then move them.

    Chunked forward: q,k [B,T,Hk,Dk]; v [B,T,Hv,Dv]; g [B,T,Hv] or [B,T,Hv,Dk];
    beta [B,T,Hv]; h0 [B,Hv,Dk,Dv] or None.
    Decode (w.decode): the leading axis is the step: q,k [T,B,Hk,Dk] ... with
    T = number of steps, and h0 [B,Hv,Dk,Dv].
    """
    gen = torch.Generator(device="cpu").manual_seed(w.seed)
    lead = (w.T, w.B) if w.decode else (w.B, w.T)
    dt = w.torch_dtype

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q = _unit(randn(*lead, w.Hk, w.Dk)).to(dt)
    k = _unit(randn(*lead, w.Hk, w.Dk)).to(dt)
    v = randn(*lead, w.Hv, w.Dv).to(dt)
    gshape = (*lead, w.Hv) if w.gate == "scalar" else (*lead, w.Hv, w.Dk)
    g = torch.nn.functional.logsigmoid(randn(*gshape) + w.g_mu)
    beta = torch.sigmoid(randn(*lead, w.Hv))
    h0 = (randn(w.B, w.Hv, w.Dk, w.Dv) * w.h0_std) if w.h0_std > 0 else None
    out = dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0)
    if device != "cpu":
        out = {n: (None if t is None else t.to(device)) for n, t in out.items()}
    return out


def make_upstream(w: Workload, device="cpu"):
    """Upstream gradients of a backward step, from a second generator seeded w.seed + 1000003:
    do ~ N(0, 1) [B, T, Hv, Dv] in the workload dtype, then dhT = 0.1 N(0, 1) [B, Hv, Dk, Dv] fp32."""
    gen = torch.Generator(device="cpu").manual_seed(w.seed + 1000003)
    do = torch.randn((w.B, w.T, w.Hv, w.Dv), generator=gen).to(w.torch_dtype)
    dhT = 0.1 * torch.randn((w.B, w.Hv, w.Dk, w.Dv), generator=gen)
    return {"do": do.to(device), "dhT": dhT.to(device)}


def make_layer_inputs(w: Workload, device="cpu"):
    """The layer around the recurrence, drawn in this order from one generator:

      xq, xk ~ N(0, 1) [B, T, Hk*Dk], xv ~ N(0, 1) [B, T, Hv*Dv] (bf16): the q/k/v
             projections before the short convolution
      wq, wk [Hk*Dk, 4], wv [Hv*Dv, 4] = 0.5 N(0, 1) (fp32): the convolution taps
      g, beta, h0 as in make_inputs
      z ~ N(0, 1) [B, T, Hv, Dv] (bf16): the output gate
      nw = 1 + 0.1 N(0, 1) [Dv] (fp32): the output norm's weight
    """
    gen = torch.Generator(device="cpu").manual_seed(w.seed)
    dt = w.torch_dtype

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    out = dict(xq=randn(w.B, w.T, w.Hk * w.Dk).to(dt), xk=randn(w.B, w.T, w.Hk * w.Dk).to(dt),
               xv=randn(w.B, w.T, w.Hv * w.Dv).to(dt))
    out.update(wq=0.5 * randn(w.Hk * w.Dk, 4), wk=0.5 * randn(w.Hk * w.Dk, 4), wv=0.5 * randn(w.Hv * w.Dv, 4))
    gshape = (w.B, w.T, w.Hv) if w.gate == "scalar" else (w.B, w.T, w.Hv, w.Dk)
    out["g"] = torch.nn.functional.logsigmoid(randn(*gshape) + w.g_mu)
    out["beta"] = torch.sigmoid(randn(w.B, w.T, w.Hv))
    out["h0"] = (randn(w.B, w.Hv, w.Dk, w.Dv) * w.h0_std) if w.h0_std > 0 else None
    out["z"] = randn(w.B, w.T, w.Hv, w.Dv).to(dt)
    out["nw"] = 1.0 + 0.1 * randn(w.Dv)
    if device != "cpu":
        out = {n: (None if t is None else t.to(device)) for n, t in out.items()}
    return out
