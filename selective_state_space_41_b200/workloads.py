"""Synthetic workloads for the selective-scan forward and their input recipes.

Each workload fixes (batch B, channels D, steps L, state size N), the input
dtype, which optional operands are present, and how every operand is drawn.
Shapes follow the selective_scan_ref layouts of the walkthrough page
("Mamba代码实战：手把手教你用PyTorch复现选择性扫描核心逻辑（附避坑指南）", §2.1 初始化参数):
u, delta, z (B, D, L); A (D, N); B, C (B, N, L); D, delta_bias (D,).

A[d, n] = -(n + 1) is the A_log = log(1..N) initialisation of the mamba-minimal
pages (A = -exp(A_log); "告别‘炼丹’：从Mamba-minimal入手..." §1.1 and
"Mamba-minimal项目解析" §5).  All other operands are seeded draws from ``gen``.
"""
import math
from dataclasses import dataclass, replace

import torch

from . import gen

# Philox stream ids, one per operand.
STREAM = {"u": 1, "delta": 2, "B": 3, "C": 4, "z": 5, "D": 6, "delta_bias": 7, "delta_r": 11, "W_dt": 12}

# dt_rank of the dt_proj form for a layer of model width d_model: the pages
# give dt_rank = 'auto' without a rule ("Mamba-minimal项目解析", 1. ModelArgs);
# read as mamba-minimal's ceil(d_model / 16) (48 for d_model 768).
def dt_rank_auto(d_model: int) -> int:
    return -(-d_model // 16)


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    dim: int
    seqlen: int
    dstate: int
    dtype: torch.dtype            # u, delta, B, C, z (and y)
    seed: int
    has_z: bool = False
    D_kind: str = "normal"        # "normal" | "ones" | "none"
    bias_kind: str = "normal"     # "normal" | "zeros" | "uniform_dt" | "none"
    delta_softplus: bool = True
    return_last_state: bool = False
    out_dtype: torch.dtype = None  # None: same as dtype

    @property
    def updates(self) -> int:
        """State updates B*D*L*N (one exp each)."""
        return self.batch * self.dim * self.seqlen * self.dstate

    def describe(self) -> dict:
        return {"workload": self.name, "batch": self.batch, "dim": self.dim,
                "seqlen": self.seqlen, "dstate": self.dstate,
                "dtype": str(self.dtype).replace("torch.", ""), "z_gate": self.has_z,
                "delta_softplus": self.delta_softplus,
                "return_last_state": self.return_last_state}


# delta_bias range of the mamba-130m-shaped layer: softplus(bias) in [1e-3, 0.1].
DT_BIAS_LO = math.log(math.expm1(1e-3))
DT_BIAS_HI = math.log(math.expm1(0.1))

WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_fp32_b4_d16_l64_n32", 4, 16, 64, 32, torch.float32, 4101,
                 D_kind="normal", bias_kind="normal", return_last_state=True),
        Workload("fp32_b32_d128_l256_n16", 32, 128, 256, 16, torch.float32, 4102,
                 D_kind="ones", bias_kind="zeros"),
        Workload("mamba130m_layer_b8_d1536_l2048_n16", 8, 1536, 2048, 16, torch.bfloat16, 4103,
                 has_z=True, D_kind="ones", bias_kind="uniform_dt"),
        Workload("genomic_100k_b4_d1024_l100000_n16", 4, 1024, 100000, 16, torch.bfloat16, 4104,
                 D_kind="ones", bias_kind="none", return_last_state=True),
        Workload("wide_state_b16_d4096_l8192_n16", 16, 4096, 8192, 16, torch.bfloat16, 410516,
                 has_z=True, D_kind="normal", bias_kind="none"),
        Workload("wide_state_b16_d4096_l8192_n32", 16, 4096, 8192, 32, torch.bfloat16, 410532,
                 has_z=True, D_kind="normal", bias_kind="none"),
        Workload("wide_state_b16_d4096_l8192_n64", 16, 4096, 8192, 64, torch.bfloat16, 410564,
                 has_z=True, D_kind="normal", bias_kind="none"),
    ]
}

TINY = "tiny_fp32_b4_d16_l64_n32"
MAMBA130M = "mamba130m_layer_b8_d1536_l2048_n16"
GENOMIC = "genomic_100k_b4_d1024_l100000_n16"


def custom(name, batch, dim, seqlen, dstate, dtype=torch.float32, seed=1, **kw) -> Workload:
    return Workload(name, batch, dim, seqlen, dstate, dtype, seed, **kw)


def with_shape(w: Workload, **kw) -> Workload:
    return replace(w, **kw)


def make_inputs(w: Workload, pin: bool = False, nthreads: int = 0) -> dict:
    """Host tensors for workload ``w`` plus its flags, keyed by argument name."""
    B, D, L, N = w.batch, w.dim, w.seqlen, w.dstate

    def draw(name, shape, dtype, kind=gen.NORMAL, p0=0.0, p1=1.0):
        return gen.fill(shape, dtype, w.seed, STREAM[name], kind, p0, p1, pin, nthreads)

    out = {
        "u": draw("u", (B, D, L), w.dtype),
        "delta": draw("delta", (B, D, L), w.dtype),
        "A": -torch.arange(1, N + 1, dtype=torch.float32).repeat(D, 1).contiguous(),
        "B": draw("B", (B, N, L), w.dtype),
        "C": draw("C", (B, N, L), w.dtype),
        "z": draw("z", (B, D, L), w.dtype) if w.has_z else None,
        "delta_softplus": w.delta_softplus,
        "return_last_state": w.return_last_state,
    }
    if w.D_kind == "normal":
        out["D"] = draw("D", (D,), torch.float32)
    elif w.D_kind == "ones":
        out["D"] = torch.ones(D, dtype=torch.float32)
    else:
        out["D"] = None
    if w.bias_kind == "normal":
        out["delta_bias"] = draw("delta_bias", (D,), torch.float32)
    elif w.bias_kind == "zeros":
        out["delta_bias"] = torch.zeros(D, dtype=torch.float32)
    elif w.bias_kind == "uniform_dt":
        out["delta_bias"] = draw("delta_bias", (D,), torch.float32, gen.UNIFORM,
                                 DT_BIAS_LO, DT_BIAS_HI)
    else:
        out["delta_bias"] = None
    if pin:
        out["A"] = out["A"].pin_memory()
        for k in ("D", "delta_bias"):
            if out[k] is not None:
                out[k] = out[k].pin_memory()
    out["out_dtype"] = w.out_dtype or w.dtype
    return out


def make_dtproj_inputs(w: Workload, dt_rank: int, pin: bool = False) -> dict:
    """make_inputs(w) plus the low-rank input of the dt_proj form: delta_r
    (B, dt_rank, L) ~ N(0, 1) and W_dt (D, dt_rank) ~ U(-dt_rank^-1/2,
    dt_rank^-1/2), both in the workload's dtype (delta = W_dt delta_r then has
    standard deviation about 0.58); delta is left out (None)."""
    out = make_inputs(w, pin=pin)
    out["delta"] = None
    bound = dt_rank ** -0.5
    out["delta_r"] = gen.fill((w.batch, dt_rank, w.seqlen), w.dtype, w.seed, STREAM["delta_r"], gen.NORMAL,
                              0.0, 1.0, pin)
    out["W_dt"] = gen.fill((w.dim, dt_rank), w.dtype, w.seed, STREAM["W_dt"], gen.UNIFORM, -bound, bound, pin)
    return out
