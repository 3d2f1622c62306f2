"""Seeded synthetic inputs for SS2D, shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and lays them out; it holds none of the
scan's arithmetic.  The value distributions follow the initialisation recipe
of the Mamba module printed on "vision mamba-yolov8" (section "2. Vmamba module
code", class Mamba.__init__):

* the step-size bias is the inverse softplus of a dt drawn log-uniformly in
  [dt_min, dt_max] = [1e-3, 1e-1] and clamped below at 1e-4;
* A follows the S4D-real initialisation, A[c, n] = -(n + 1) (kept in fp32 as
  -exp(log(n + 1)));
* the skip parameter D is 1.

Shapes follow VMamba-T (dim 96, ssm_ratio 2 -> D = 192 channels, d_state 16) at
a 224x224 input: stage 1 is a 56x56 map, stage 3 a 14x14 map with 768
channels.  u, delta, B, C are drawn in fp32 and rounded to bf16 (round to
nearest even) for the bf16 workloads; A, D and the bias stay fp32.

Draw order from one torch.Generator seeded with the workload index:
u, delta, B, C, dt, dy.  The same seed on another device gives other values
(torch's CPU and CUDA generators differ); every consumer receives the tensors
themselves, so the oracle and the kernels always see identical numbers.

The bidirectional scan (bimamba_inner_ref on the same page) takes a sequence of
tokens.  Its workload follows the VisionMamba call printed on "Vision Mamba架构深入解析"
(jsqmd.com), section "双向状态空间模型设计" (bidirectional state-space model design):
img_size=224, patch_size=16, embed_dim=192, so 14 x 14 = 196 patch tokens plus
a class token, L = 197, and an inner width of 2 x 192 = 384 channels (the
Mamba block's default expansion of 2), d_state 16.  Its A and A_b both follow
the S4D-real initialisation; tests may ask for A_b scaled elementwise by a
seeded factor in [0.5, 1.5] so that the two directions differ.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

K_PATHS = 4


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    dim: int          # D, channels per path
    height: int
    width: int
    d_state: int      # N
    dtype: str        # "f32" or "bf16": dtype of u, delta, B, C and the output
    a_init: str       # "neg_index": A = -(n+1) exactly; "s4d_real": -exp(log(n+1)) in fp32
    backward: bool = False
    description: str = ""
    kind: str = "ss2d"  # "ss2d": four paths over an H x W map; "bidir": a sequence and its reverse

    @property
    def L(self) -> int:
        return self.height * self.width

    @property
    def paths(self) -> int:
        return 2 if self.kind == "bidir" else K_PATHS

    @property
    def channels(self) -> int:
        return self.paths * self.dim

    @property
    def updates(self) -> int:
        """state updates of one forward: B * paths * D * L * N"""
        return self.batch * self.paths * self.dim * self.L * self.d_state

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_batch(self, batch: int) -> "Workload":
        return replace(self, batch=batch)


WORKLOADS = [
    Workload("tiny_fp32", 1, 8, 8, 8, 4, "f32", "neg_index",
             description="tiny SS2D fwd, B=1 D=8 H=W=8 (L=64) N=4, fp32"),
    Workload("vmamba_t_stage1_fp32", 128, 192, 56, 56, 16, "f32", "s4d_real",
             description="VMamba-T stage-1 SS2D fwd, B=128 D=192 H=W=56 (L=3136) N=16, fp32"),
    Workload("vmamba_stage3_bf16", 128, 768, 14, 14, 16, "bf16", "s4d_real",
             description="VMamba stage-3 SS2D fwd, B=128 D=768 H=W=14 (L=196) N=16, bf16 in / fp32 state"),
    Workload("highres_128_bf16", 8, 192, 128, 128, 16, "bf16", "s4d_real",
             description="high-resolution SS2D fwd, B=8 D=192 H=W=128 (L=16384) N=16, bf16 in / fp32 state"),
    Workload("vmamba_t_stage1_fwd_bwd_fp32", 32, 192, 56, 56, 16, "f32", "s4d_real", backward=True,
             description="SS2D fwd+bwd, B=32 D=192 H=W=56 N=16, fp32, dy ~ N(0,1)"),
    Workload("vim_t_bidir_fp32", 128, 384, 1, 197, 16, "f32", "s4d_real", kind="bidir",
             description="bidirectional scan (Vim-T tokens), B=128 D=384 L=197 N=16, fp32, gate z"),
]


def workload(index_or_name) -> Workload:
    if isinstance(index_or_name, int):
        return WORKLOADS[index_or_name]
    for w in WORKLOADS:
        if w.name == index_or_name:
            return w
    raise KeyError(index_or_name)


def custom(batch, dim, height, width, d_state, dtype="f32", a_init="neg_index", backward=True, kind="ss2d"):
    return Workload(f"custom_{kind}_{batch}x{dim}x{height}x{width}_n{d_state}_{dtype}", batch, dim, height,
                    width, d_state, dtype, a_init, backward, kind=kind)


def make_inputs(w: Workload, seed: int = 0, device="cpu", with_dy: bool | None = None):
    """Draw one SS2D problem.  Returns a dict of tensors on `device`:

    x (B, D, H, W), delta (B, 4D, L), A (4D, N) fp32, B and C (B, 4, N, L),
    D (4D) fp32, delta_bias (4D) fp32 and, when asked, dy (B, D, H, W).
    """
    if with_dy is None:
        with_dy = w.backward
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    f32 = dict(dtype=torch.float32, device=device, generator=g)
    Bn, Dn, L, N = w.batch, w.dim, w.L, w.d_state
    x = torch.randn((Bn, Dn, w.height, w.width), **f32)
    delta = torch.randn((Bn, K_PATHS * Dn, L), **f32) * 0.1
    Bm = torch.randn((Bn, K_PATHS, N, L), **f32)
    Cm = torch.randn((Bn, K_PATHS, N, L), **f32)
    dt_min, dt_max, dt_floor = 1e-3, 1e-1, 1e-4
    dt = torch.exp(torch.rand((K_PATHS * Dn,), **f32) * (math.log(dt_max) - math.log(dt_min))
                   + math.log(dt_min)).clamp(min=dt_floor)
    delta_bias = dt + torch.log(-torch.expm1(-dt))
    n1 = torch.arange(1, N + 1, dtype=torch.float32, device=device)
    if w.a_init == "neg_index":
        A_row = -n1
    else:
        A_row = -torch.exp(torch.log(n1))
    A = A_row.unsqueeze(0).repeat(K_PATHS * Dn, 1).contiguous()
    Dv = torch.ones(K_PATHS * Dn, dtype=torch.float32, device=device)
    out = dict(x=x, delta=delta, A=A, B=Bm, C=Cm, D=Dv, delta_bias=delta_bias)
    if with_dy:
        out["dy"] = torch.randn((Bn, Dn, w.height, w.width), **f32)
    if w.dtype == "bf16":
        for key in ("x", "delta", "B", "C", "dy"):
            if key in out:
                out[key] = out[key].to(torch.bfloat16)
    return out


def make_bimamba_inputs(w: Workload, seed: int = 0, device="cpu", with_dy: bool = False, with_z: bool = False,
                        distinct_a_b: bool = False):
    """Draw one bidirectional-scan problem (w.kind == "bidir", w.height == 1).  Returns x, delta,
    z (B, D, L); A, A_b (D, N) fp32; B, C (B, N, L); D, delta_bias (D) fp32; dy (B, D, L) if asked.
    Draw order: x, delta, B, C, dt, [z], [dy], [A_b factor]."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) + 2000)
    f32 = dict(dtype=torch.float32, device=device, generator=g)
    Bn, Dn, L, N = w.batch, w.dim, w.L, w.d_state
    x = torch.randn((Bn, Dn, L), **f32)
    delta = torch.randn((Bn, Dn, L), **f32) * 0.1
    Bm = torch.randn((Bn, N, L), **f32)
    Cm = torch.randn((Bn, N, L), **f32)
    dt_min, dt_max, dt_floor = 1e-3, 1e-1, 1e-4
    dt = torch.exp(torch.rand((Dn,), **f32) * (math.log(dt_max) - math.log(dt_min))
                   + math.log(dt_min)).clamp(min=dt_floor)
    delta_bias = dt + torch.log(-torch.expm1(-dt))
    n1 = torch.arange(1, N + 1, dtype=torch.float32, device=device)
    A_row = -n1 if w.a_init == "neg_index" else -torch.exp(torch.log(n1))
    A = A_row.unsqueeze(0).repeat(Dn, 1).contiguous()
    out = dict(x=x, delta=delta, A=A, A_b=A.clone(), B=Bm, C=Cm, D=torch.ones(Dn, dtype=torch.float32, device=device),
               delta_bias=delta_bias)
    if with_z:
        out["z"] = torch.randn((Bn, Dn, L), **f32)
    if with_dy:
        out["dy"] = torch.randn((Bn, Dn, L), **f32)
    if distinct_a_b:
        out["A_b"] = (A * (0.5 + torch.rand((Dn, N), **f32))).contiguous()
    if w.dtype == "bf16":
        for key in ("x", "delta", "B", "C", "z", "dy"):
            if key in out:
                out[key] = out[key].to(torch.bfloat16)
    return out


def dt_rank_of(dim: int) -> int:
    """dt_rank = ceil(d_model / 16) (Mamba.__init__), with d_model = dim / 2 for SS2D's
    expansion of 2 (VMamba-T: 192 channels, d_model 96, rank 6)."""
    return max(1, math.ceil((dim // 2) / 16))


def make_proj_inputs(w: Workload, seed: int = 0, device="cpu", d_conv: int = 0):
    """Inputs of the SS2D forward with its producer (x_proj, dt_proj per path), drawn as
    Mamba.__init__ initialises them: x ~ N(0,1) (B, D, H, W); x_proj weight (4, R+2N, D)
    ~ U(-1/sqrt(D), 1/sqrt(D)) (nn.Linear's default); dt_proj weight (4, D, R) ~
    U(-R^-0.5, R^-0.5) (dt_init "random", dt_scale 1); dt_proj bias, A and D as in make_inputs.
    Draw order: x, x_proj weight, dt_proj weight, dt.  With d_conv > 0, the per-path causal
    depthwise conv follows, as nn.Conv1d(D, D, d_conv, groups=D) initialises it: weight (4, D,
    d_conv) and bias (4D), both ~ U(-1/sqrt(d_conv), 1/sqrt(d_conv)), drawn after the rest."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) + 3000)
    f32 = dict(dtype=torch.float32, device=device, generator=g)
    Bn, Dn, N = w.batch, w.dim, w.d_state
    R = dt_rank_of(Dn)
    x = torch.randn((Bn, Dn, w.height, w.width), **f32)
    bx = 1.0 / math.sqrt(Dn)
    Wx = (torch.rand((K_PATHS, R + 2 * N, Dn), **f32) * 2 - 1) * bx
    bd = R ** -0.5
    Wdt = (torch.rand((K_PATHS, Dn, R), **f32) * 2 - 1) * bd
    dt_min, dt_max, dt_floor = 1e-3, 1e-1, 1e-4
    dt = torch.exp(torch.rand((K_PATHS * Dn,), **f32) * (math.log(dt_max) - math.log(dt_min))
                   + math.log(dt_min)).clamp(min=dt_floor)
    bias = dt + torch.log(-torch.expm1(-dt))
    n1 = torch.arange(1, N + 1, dtype=torch.float32, device=device)
    A_row = -n1 if w.a_init == "neg_index" else -torch.exp(torch.log(n1))
    A = A_row.unsqueeze(0).repeat(K_PATHS * Dn, 1).contiguous()
    out = dict(x=x, x_proj_weight=Wx, dt_proj_weight=Wdt, dt_proj_bias=bias, A=A,
               D=torch.ones(K_PATHS * Dn, dtype=torch.float32, device=device), R=R)
    if d_conv > 0:
        bc = 1.0 / math.sqrt(d_conv)
        out["conv_weight"] = (torch.rand((K_PATHS, Dn, d_conv), **f32) * 2 - 1) * bc
        out["conv_bias"] = (torch.rand((K_PATHS * Dn,), **f32) * 2 - 1) * bc
    if w.dtype == "bf16":
        out["x"] = out["x"].to(torch.bfloat16)
    return out


def batch_slice(inputs: dict, idx) -> dict:
    """Restrict batch-indexed tensors to batch items `idx` (a list); parameters are shared."""
    out = {}
    for k, v in inputs.items():
        if k in ("x", "delta", "B", "C", "dy", "z", "u", "dout"):
            out[k] = v[idx]
        else:
            out[k] = v
    return out


def make_scan_inputs(w: Workload, seed: int = 0, device="cpu", with_dout: bool = False, with_z: bool = False):
    """Inputs for the standalone S6 scan in its sequence view: u (B, 4D, L) drawn directly
    (N(0,1)) instead of an image, the other tensors as in make_inputs.  dout ~ N(0,1) if asked;
    the output gate z ~ N(0,1) (B, 4D, L) if asked, drawn last so the other tensors do not change."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) + 1000)
    f32 = dict(dtype=torch.float32, device=device, generator=g)
    base = make_inputs(w, seed=seed, device=device, with_dy=False)
    u = torch.randn((w.batch, K_PATHS * w.dim, w.L), **f32)
    out = dict(base)
    del out["x"]
    out["u"] = u
    if with_dout:
        out["dout"] = torch.randn((w.batch, K_PATHS * w.dim, w.L), **f32)
    if with_z:
        out["z"] = torch.randn((w.batch, K_PATHS * w.dim, w.L), **f32)
    if w.dtype == "bf16":
        for key in ("u", "dout", "z"):
            if key in out:
                out[key] = out[key].to(torch.bfloat16)
    return out
