"""Seeded synthetic inputs for the TTT layer forward.

This module only draws random numbers; it holds none of the layer's arithmetic.  Both the CUDA
path (tests, bench) and the fp64 oracle read the very same tensors produced here.

Recipe (one torch CPU generator, ``manual_seed(seed)``, float32 draws in this order):
  Q, K, V  : [B][heads][N][d] standard normal; every q and k row (length d) is then divided by its
             L2 norm (keys and queries are L2-normalised rows, values stay N(0, 1));
  weights  : linear W0 [heads_lin][d][d] ~ N(0, 1/d); conv W0 [heads_conv][d][3][3] ~ N(0, 1/9);
             full 3x3 conv W0 [heads][d][d][3][3] ~ N(0, 1/(9d)) (its fan-in is 9d);
             MLP Wa [heads][4d][d] ~ N(0, 1/d), Wb [heads][d][4d] ~ N(0, 1/(4d));
  dZ       : (kind "backward", the upstream gradient of Z) [B][heads][N][d] standard normal, drawn
             after the weights;
then Q, K, V (and dZ) are rounded once to the compute dtype (bf16: round-to-nearest-even) and
weights stay float32.  Token n of a unit sits at grid position (n // W, n % W) (raster order of the 16x16
patches of the image).

Workloads (token counts are the pages' image sizes divided into 16 x 16 patches:
224^2 -> 14 x 14 = 196, 1248^2 -> 78 x 78 = 6084, 1280^2 -> 80 x 80 = 6400):
  lin196_fp32      linear, B 1,  1 head, 14 x 14, fp32, eta 1.0
  lin196_bf16      linear, B 64, 3 heads, 14 x 14, bf16, eta 1.0   (ViT-Tiny-shaped 224^2 layer)
  mixed6084_bf16   5 linear heads + 1 depthwise-conv head (the last head), B 8, 78 x 78, bf16, eta 0.5
  lin6400_bf16     linear, B 4, 12 heads, 80 x 80, bf16, eta 1.0   (ViT-Base-shaped 1280^2 layer)
  mlp1024_bf16     MLP width 4d = 256, GELU(tanh), B 16, 4 heads, 32 x 32, bf16, eta 0.5
  mixed6084_dot_bf16  as mixed6084_bf16, trained with the dot-product inner loss and eta 1.0 (the
                   ViT3 recipe: one full-batch step, learning rate 1.0, dot-product loss)
  mb16_6084_bf16   linear, B 8, 6 heads, 78 x 78, bf16, trained by mini-batch gradient descent in
                   consecutive batches of 16 tokens (causal prefix inside a batch), eta 0.25
  bwd6084_bf16     backward pass of the linear heads of mixed6084_bf16: B 8, 5 heads, 78 x 78,
                   bf16, eta 0.5
  bwdconv6084_bf16 backward pass of the depthwise-conv head of mixed6084_bf16: B 8, 1 head, 78 x 78,
                   bf16, eta 0.5 (conv W0 and dZ as above)
  bwdmlp1024_bf16  backward pass of mlp1024_bf16's MLP head: B 16, 4 heads, 32 x 32, bf16, eta 0.5
  conv3x3_6084_bf16  the full 3x3 conv head (the press article's other conv variant) in place of the
                   depthwise head of mixed6084_bf16: B 8, 1 head, 78 x 78, bf16, eta 0.5
"""
from dataclasses import dataclass
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int            # total heads of the layer
    H: int                # token grid height
    W: int                # token grid width
    dtype: str            # "fp32" or "bf16"
    eta: float
    kind: str             # "linear", "mixed" (linear heads + conv heads last), "mlp", "minibatch" (linear),
                          # "backward" (linear), "backward_conv" (depthwise conv), "backward_mlp" (MLP),
                          # "conv3x3" (full 3x3 conv heads)
    conv_heads: int = 0   # number of depthwise-conv heads (the last ones) for "mixed"
    d: int = 64
    hidden_ratio: int = 4
    loss: str = "l2"      # inner loss: "l2" or "dot"
    mb_tokens: int = 0    # kind "minibatch": tokens per mini-batch
    mb_mode: str = "prefix"

    @property
    def N(self):
        return self.H * self.W

    @property
    def lin_heads(self):
        return self.heads - self.conv_heads if self.kind in ("linear", "mixed", "minibatch", "backward") else 0

    @property
    def token_heads(self):
        return self.batch * self.heads * self.N


WORKLOADS = {
    "lin196_fp32": Workload("lin196_fp32", 1, 1, 14, 14, "fp32", 1.0, "linear"),
    "lin196_bf16": Workload("lin196_bf16", 64, 3, 14, 14, "bf16", 1.0, "linear"),
    "mixed6084_bf16": Workload("mixed6084_bf16", 8, 6, 78, 78, "bf16", 0.5, "mixed", conv_heads=1),
    "lin6400_bf16": Workload("lin6400_bf16", 4, 12, 80, 80, "bf16", 1.0, "linear"),
    "mlp1024_bf16": Workload("mlp1024_bf16", 16, 4, 32, 32, "bf16", 0.5, "mlp"),
    "mixed6084_dot_bf16": Workload("mixed6084_dot_bf16", 8, 6, 78, 78, "bf16", 1.0, "mixed", conv_heads=1,
                                   loss="dot"),
    "mb16_6084_bf16": Workload("mb16_6084_bf16", 8, 6, 78, 78, "bf16", 0.25, "minibatch", mb_tokens=16),
    "bwd6084_bf16": Workload("bwd6084_bf16", 8, 5, 78, 78, "bf16", 0.5, "backward"),
    "bwdconv6084_bf16": Workload("bwdconv6084_bf16", 8, 1, 78, 78, "bf16", 0.5, "backward_conv", conv_heads=1),
    "bwdmlp1024_bf16": Workload("bwdmlp1024_bf16", 16, 4, 32, 32, "bf16", 0.5, "backward_mlp"),
    "conv3x3_6084_bf16": Workload("conv3x3_6084_bf16", 8, 1, 78, 78, "bf16", 0.5, "conv3x3"),
}

TORCH_DTYPE = {"fp32": torch.float32, "bf16": torch.bfloat16}


def _unit_rows(x):
    return x / x.norm(dim=-1, keepdim=True)


def make_inputs(w: Workload, seed: int = 0, device="cpu"):
    """Returns a dict of tensors: Q, K, V (compute dtype) and the fp32 weights of the workload."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (w.batch, w.heads, w.N, w.d)
    Q = _unit_rows(torch.randn(shape, generator=g, dtype=torch.float32))
    K = _unit_rows(torch.randn(shape, generator=g, dtype=torch.float32))
    V = torch.randn(shape, generator=g, dtype=torch.float32)
    out = {}
    if w.kind in ("linear", "mixed", "minibatch", "backward", "backward_conv"):
        if w.lin_heads:
            out["W0_lin"] = torch.randn((w.lin_heads, w.d, w.d), generator=g) / math.sqrt(w.d)
        if w.conv_heads:
            out["W0_conv"] = torch.randn((w.conv_heads, w.d, 3, 3), generator=g) / 3.0
    elif w.kind == "conv3x3":
        out["W0_c3"] = torch.randn((w.heads, w.d, w.d, 3, 3), generator=g) / math.sqrt(9 * w.d)
    elif w.kind in ("mlp", "backward_mlp"):
        hid = w.hidden_ratio * w.d
        out["Wa"] = torch.randn((w.heads, hid, w.d), generator=g) / math.sqrt(w.d)
        out["Wb"] = torch.randn((w.heads, w.d, hid), generator=g) / math.sqrt(hid)
    dt = TORCH_DTYPE[w.dtype]
    if w.kind in ("backward", "backward_conv", "backward_mlp"):
        out["dZ"] = torch.randn(shape, generator=g, dtype=torch.float32).to(dt)
    out["Q"], out["K"], out["V"] = Q.to(dt), K.to(dt), V.to(dt)
    if device != "cpu":
        out = {k: v.to(device) for k, v in out.items()}
    return out


def random_unit(batch, heads, H, W, d=64, dtype="bf16", seed=0, kind="linear", conv_heads=0,
                hidden_ratio=4, eta=1.0):
    """Inputs for an arbitrary (test) shape with the same distributions."""
    w = Workload("custom", batch, heads, H, W, dtype, eta, kind, conv_heads=conv_heads, d=d,
                 hidden_ratio=hidden_ratio)
    return w, make_inputs(w, seed)
