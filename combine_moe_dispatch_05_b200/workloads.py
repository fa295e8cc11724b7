"""Seeded synthetic inputs for MoE token dispatch / combine.

This module only draws random numbers with the shapes and distributions of the
workloads below.  It holds none of the dispatch/combine arithmetic: no counting,
no prefix sums, no row placement, no reductions, no quantisation.  Both the CUDA
path and the CPU oracle are fed from here, so neither one generates the other's
inputs.

Workloads (sizes follow the DeepSeek-V3-like shapes H=7168, E=256, K=8 used for
the decode and prefill cases; the serving traces the pages evaluate on are not
available, so these seeded routings stand in for them):

  1 tiny     T=256   H=128  E=8   K=2 R=2   uniform distinct ids, x ~ U[-1,1]
  2 decode   T=4096  H=7168 E=256 K=8 R=8   Zipf(s=0.6) ids, x ~ N(0,1)
  3 prefill  T=32768 H=7168 E=256 K=8 R=8   Zipf(s=1.2) ids, x ~ N(0,1) (FP8 path)
  4 shared   T=8192  H=4096 E=64  K=6 R=16  uniform distinct ids, y, shared ~ N(0,0.5)
  5 bwd      T=16384 H=4096 E=8   K=2 R=1   one hot expert in 60% of tokens' top-2
                                            (the "100% hot" variant puts it in every row)

Expert ids within a row are distinct (the Ascend combine API's expert_ids
contract: values in [0, moe_expert_num), no repeats within a row).  Distinct
ids with a popularity law are drawn with the Gumbel-top-K trick, which is
sequential weighted sampling without replacement; the order inside a row is
descending perturbed key.  Scales are a softmax of N(0,1) logits over the K
chosen experts.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

SEED_BASE = 20260000

# One sub-stream per tensor kind, so adding a tensor never shifts the others.
_STREAM = {"ids": 1, "scales": 2, "x": 3, "y": 4, "shared": 5, "grad": 6,
           "codes": 7, "xscales": 8, "perm": 9, "hot": 10}


@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    T: int
    H: int
    E: int
    K: int
    R: int
    routing: str              # "uniform" | "zipf" | "hot"
    zipf_s: float = 0.0
    hot_p: float = 0.0        # probability that the hot expert is in a row
    x_dist: str = "normal"    # "uniform" (U[-1,1]) | "normal"
    sigma: float = 1.0        # std of the normal draws (x, y, shared, grad)
    seed: int = SEED_BASE

    def with_(self, **kw) -> "Spec":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    1: Spec("tiny", 256, 128, 8, 2, 2, "uniform", x_dist="uniform", seed=SEED_BASE + 1),
    2: Spec("dsv3_decode", 4096, 7168, 256, 8, 8, "zipf", zipf_s=0.6, seed=SEED_BASE + 2),
    3: Spec("prefill_fp8", 32768, 7168, 256, 8, 8, "zipf", zipf_s=1.2, seed=SEED_BASE + 3),
    4: Spec("shared_expert", 8192, 4096, 64, 6, 16, "uniform", sigma=0.5, seed=SEED_BASE + 4),
    5: Spec("bwd_skew", 16384, 4096, 8, 2, 1, "hot", hot_p=0.6, seed=SEED_BASE + 5),
}


def config(i: int, seed_offset: int = 0) -> Spec:
    s = CONFIGS[i]
    return s.with_(seed=s.seed + 1000 * seed_offset) if seed_offset else s


def _gen(spec: Spec, kind: str, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(spec.seed * 64 + _STREAM[kind])
    return g


def topk_ids(spec: Spec) -> torch.Tensor:
    """int32 [T, K] expert ids, distinct within each row."""
    T, E, K = spec.T, spec.E, spec.K
    g = _gen(spec, "ids")
    if spec.routing == "hot":
        return _hot_ids(spec, g)
    if spec.routing == "uniform":
        logw = torch.zeros(E, dtype=torch.float64)
    elif spec.routing == "zipf":
        # popularity p_{pi(i)} ~ (i+1)^-s over a seeded permutation pi of the experts
        perm = torch.randperm(E, generator=_gen(spec, "perm"))
        rank_of = torch.empty(E, dtype=torch.float64)
        rank_of[perm] = torch.arange(1, E + 1, dtype=torch.float64)
        logw = -spec.zipf_s * torch.log(rank_of)
    else:
        raise ValueError(spec.routing)
    ids = torch.empty((T, K), dtype=torch.int32)
    chunk = max(1, (1 << 22) // max(E, 1))
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        u = torch.rand((t1 - t0, E), generator=g, dtype=torch.float64)
        u.clamp_(min=1e-300)
        gumbel = -torch.log(-torch.log(u))
        keys = logw.unsqueeze(0) + gumbel
        ids[t0:t1] = torch.topk(keys, K, dim=1, sorted=True).indices.to(torch.int32)
    return ids


def _hot_ids(spec: Spec, g: torch.Generator) -> torch.Tensor:
    """One seeded hot expert appears in a row with probability hot_p, at a random
    position; the remaining slots are uniform over the other experts, without
    replacement."""
    T, E, K = spec.T, spec.E, spec.K
    hot = int(torch.randint(E, (1,), generator=_gen(spec, "hot")).item())
    others = torch.tensor([e for e in range(E) if e != hot], dtype=torch.int64)
    u = torch.rand((T, E - 1), generator=g, dtype=torch.float64)
    pick = torch.topk(u, K, dim=1, sorted=True).indices  # K distinct non-hot experts
    ids = others[pick]
    has_hot = torch.rand((T,), generator=g, dtype=torch.float64) < spec.hot_p
    pos = torch.randint(K, (T,), generator=g)
    rows = torch.nonzero(has_hot).flatten()
    ids[rows, pos[rows]] = hot
    return ids.to(torch.int32)


def hot_expert(spec: Spec) -> int:
    return int(torch.randint(spec.E, (1,), generator=_gen(spec, "hot")).item())


def topk_scales(spec: Spec) -> torch.Tensor:
    """float32 [T, K]: softmax over the K chosen experts of N(0,1) logits."""
    g = _gen(spec, "scales")
    logits = torch.randn((spec.T, spec.K), generator=g, dtype=torch.float32)
    return torch.softmax(logits, dim=1).contiguous()


def _bf16_rows(spec: Spec, kind: str, rows: int, cols: int, dist: str, sigma: float,
               device="cpu") -> torch.Tensor:
    g = _gen(spec, kind, device)
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device=device)
    step = max(1, (1 << 24) // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        if dist == "uniform":
            blk = torch.rand((r1 - r0, cols), generator=g, dtype=torch.float32, device=device) * 2 - 1
        else:
            blk = torch.randn((r1 - r0, cols), generator=g, dtype=torch.float32, device=device) * sigma
        out[r0:r1] = blk.to(torch.bfloat16)
    return out


def tokens(spec: Spec, device="cpu") -> torch.Tensor:
    """bf16 [T, H] token activations x."""
    return _bf16_rows(spec, "x", spec.T, spec.H, spec.x_dist, spec.sigma, device)


def expert_out(spec: Spec, rows: int, device="cpu") -> torch.Tensor:
    """bf16 [rows, H] expert outputs y (rows = the caller's padded capacity)."""
    return _bf16_rows(spec, "y", rows, spec.H, "normal", spec.sigma, device)


def shared_out(spec: Spec, device="cpu") -> torch.Tensor:
    """bf16 [T, H] shared-expert output."""
    return _bf16_rows(spec, "shared", spec.T, spec.H, "normal", spec.sigma, device)


def grad_out(spec: Spec, device="cpu") -> torch.Tensor:
    """bf16 [T, H] upstream gradient of the combine output."""
    return _bf16_rows(spec, "grad", spec.T, spec.H, "normal", spec.sigma, device)


def e4m3_codes(spec: Spec, device="cpu") -> torch.Tensor:
    """uint8 [T, H] random E4M3 byte codes, NaN codes (0x7F, 0xFF) excluded."""
    g = _gen(spec, "codes", device)
    c = torch.randint(0, 254, (spec.T, spec.H), generator=g, dtype=torch.int32, device=device)
    c = c + (c >= 0x7F).to(torch.int32)          # skip 0x7F
    return c.to(torch.uint8)                     # 0..254 except 0x7F -> never 0xFF


def block_scales(spec: Spec, device="cpu") -> torch.Tensor:
    """float32 [T, H/128] positive per-128-channel scales (random, for byte-copy tests)."""
    g = _gen(spec, "xscales", device)
    return torch.rand((spec.T, spec.H // 128), generator=g, dtype=torch.float32,
                      device=device) * 0.01 + 1e-4


def as_u16(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bits of a CPU tensor as a uint16 numpy array (no copy when possible)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_u16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
