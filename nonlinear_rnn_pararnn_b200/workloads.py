"""Seeded synthetic workloads for the Newton-solved diag-mix sLSTM.

This module draws inputs only.  It holds none of the method's arithmetic and
is the one piece shared by the tests, the benchmark and the CPU oracle's
callers: both sides of every parity check receive the same arrays from here.

Distributions (one seeded ``torch.Generator`` on the CPU per workload; draw
order x, W_x, R, then dH):
  x    ~ N(0, 1)                        shape (B, T, d_in)
  W_x  ~ N(0, 1/d_in)  (std d_in^-1/2)  shape (4 d_h, d_in), rows gate-major
  R    ~ U(-a, a)                       shape (4, d_h), a = 0.5 or 0.3
  bias: b_z = b_i = b_o = 0, b_f = linspace(3, 6, d_h) (inclusive endpoints)
  s0 = 0                                shape (B, 4, d_h)
  dH   ~ N(0, 1)                        shape (B, T, d_h)
For bf16 workloads x and W_x are drawn in fp32 and rounded once to bf16
(round to nearest even); everything else stays fp32.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    d_in: int
    d_h: int
    dtype: str            # "f32" or "bf16": storage type of x and W_x
    forget: str           # "sigmoid" or "exp"
    r_scale: float        # R ~ U(-r_scale, r_scale)
    seed: int
    tol: float            # scaled-residual tolerance of the converged run
    max_iters: int        # iteration cap of the converged run
    fixed_iters: tuple = field(default=())  # fixed-K runs, if any

    @property
    def elems(self) -> int:
        return self.B * self.T * self.d_h

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "T": self.T, "d_in": self.d_in,
                "d_h": self.d_h, "x_dtype": self.dtype, "forget": self.forget,
                "tol": self.tol, "max_iters": self.max_iters, "seed": self.seed}


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 2, 64, 8, 8, "f32", "sigmoid", 0.5, 0, 1e-6, 64),
    "slstm_f32_b8_t1024_d256": Workload("slstm_f32_b8_t1024_d256", 8, 1024, 256, 256, "f32",
                                        "sigmoid", 0.5, 1, 1e-5, 1024, (3,)),
    "slstm_bf16_expgates_b16_t4096_d1024": Workload("slstm_bf16_expgates_b16_t4096_d1024", 16, 4096,
                                                    1024, 1024, "bf16", "exp", 0.5, 2, 1e-4, 8),
    "slstm_bf16_long_b4_t65536_d2048": Workload("slstm_bf16_long_b4_t65536_d2048", 4, 65536, 2048,
                                                2048, "bf16", "sigmoid", 0.3, 3, 1e-5, 16, (4,)),
    "slstm_bf16_train_b8_t8192_d1024": Workload("slstm_bf16_train_b8_t8192_d1024", 8, 8192, 1024,
                                                1024, "bf16", "sigmoid", 0.5, 4, 1e-5, 16),
}

# The five workloads in the order the specification lists them.
ORDER = list(WORKLOADS)


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (e.g. a shorter T)."""
    d = dict(w.__dict__)
    d.update(kw)
    return Workload(**d)


def make_inputs(w: Workload, with_dH: bool = True) -> dict:
    """Draw the workload's inputs on the CPU.  Returns torch tensors:
    x (B,T,d_in) and Wx (4d_h,d_in) in the workload dtype; R (4,d_h), bias
    (4,d_h), s0 (B,4,d_h) and dH (B,T,d_h) in fp32."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    x = torch.randn(w.B, w.T, w.d_in, generator=g, dtype=torch.float32)
    Wx = torch.randn(4 * w.d_h, w.d_in, generator=g, dtype=torch.float32) * (w.d_in ** -0.5)
    R = (torch.rand(4, w.d_h, generator=g, dtype=torch.float32) * 2.0 - 1.0) * w.r_scale
    dH = torch.randn(w.B, w.T, w.d_h, generator=g, dtype=torch.float32) if with_dH else None
    if w.dtype == "bf16":
        x = x.to(torch.bfloat16)
        Wx = Wx.to(torch.bfloat16)
    elif w.dtype != "f32":
        raise ValueError(w.dtype)
    bias = torch.zeros(4, w.d_h, dtype=torch.float32)
    bias[2] = torch.linspace(3.0, 6.0, w.d_h, dtype=torch.float32)
    s0 = torch.zeros(w.B, 4, w.d_h, dtype=torch.float32)
    return {"x": x, "Wx": Wx, "R": R, "bias": bias, "s0": s0, "dH": dH}


def make_head_R(w: Workload, d_head: int, seed: int = None) -> torch.Tensor:
    """Block-diagonal recurrent weights (4, d_h / d_head, d_head, d_head) for
    head mixing: entries U(-r, r) with r = the workload's R scale / sqrt(d_head),
    so that a head's recurrent input has the diagonal workloads' magnitude."""
    if w.d_h % d_head:
        raise ValueError(f"d_head={d_head} does not divide d_h={w.d_h}")
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed + 1 if seed is None else seed)
    H = w.d_h // d_head
    return (torch.rand(4, H, d_head, d_head, generator=g, dtype=torch.float32) * 2.0 - 1.0) * (w.r_scale / d_head ** 0.5)


def as_f64(t: torch.Tensor):
    """Exact widening of an fp32/bf16 tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()
