"""Seeded synthetic workloads for Selective Head Attention decode.

This module only draws random inputs and describes shapes; it holds none of
the method's arithmetic.  Both the float64 oracle (through the tests) and the
CUDA path read the same tensors made here.

Shapes follow the models the Polar Sparsity pages evaluate (OPT-66B,
LLaMA-2-7B, LLaMA-3.1-70B; papernotes.org summary, ablation table "Batch=1 /
大 Batch 加速") at the pages' batch 64 / sequence 1920 operating point
(atlas.scime.ai summary).  Values are N(0,1) stand-ins for real activations:
no model weights or datasets are used.

Seeds: Q, K and V come from one generator seeded with ``seed`` (drawn in that
order); the head index comes from a separate CPU generator seeded with
``seed + 7`` so it is reproducible on the host whatever device holds Q/K/V.
"""
from dataclasses import dataclass, replace

import torch

# Bit patterns pre-filled into inactive output rows: quiet NaNs with a payload
# no arithmetic produces, compared bit for bit.
SENTINEL = {"fp16": 0x7E5A, "bf16": 0x7FA5}
TORCH_DTYPE = {"fp16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H_q: int
    H_kv: int
    N_kv: int
    d: int
    top_k: int
    dtype: str = "fp16"
    index: str = "perm"       # "perm": first top_k of a per-row permutation; "zipf"
    seed: int = 0

    @property
    def G(self):
        return self.H_q // self.H_kv

    @property
    def units(self):
        return self.B * self.top_k

    @property
    def scale(self):
        return 1.0 / (self.d ** 0.5)

    def with_(self, **kw):
        return replace(self, **kw)

    def algorithmic_bytes(self):
        """Bytes the method must move: active K+V, active Q rows read, active O rows
        written, and the index."""
        es = 2
        return (self.units * 2 * self.N_kv * self.d * es
                + 2 * self.units * self.G * self.d * es
                + 4 * self.units)

    def flops(self):
        return 4 * self.units * self.G * self.N_kv * self.d

    def describe(self):
        return {"workload": self.name, "B": self.B, "H_q": self.H_q, "H_kv": self.H_kv,
                "N_kv": self.N_kv, "d": self.d, "top_k": self.top_k,
                "density": round(self.top_k / self.H_kv, 4), "dtype": self.dtype,
                "index": self.index, "seed": self.seed}


CONFIGS = {
    # tiny multi-head case the oracle finishes instantly
    "tiny_mha": Workload("tiny_mha", B=2, H_q=4, H_kv=4, N_kv=128, d=64, top_k=2,
                         dtype="fp16", index="perm", seed=0),
    # OPT-66B-shaped multi-head decode, about 30 % head density
    "opt66b": Workload("opt66b", B=64, H_q=72, H_kv=72, N_kv=1920, d=128, top_k=22,
                       dtype="fp16", index="perm", seed=1000),
    # the same shape with every head active (layer 0 runs dense)
    "opt66b_dense": Workload("opt66b_dense", B=64, H_q=72, H_kv=72, N_kv=1920, d=128,
                             top_k=72, dtype="fp16", index="perm", seed=1001),
    # LLaMA-2-7B-shaped decode, 50 % density, Zipf-like head popularity
    "llama2_7b": Workload("llama2_7b", B=128, H_q=32, H_kv=32, N_kv=2048, d=128,
                          top_k=16, dtype="fp16", index="zipf", seed=2000),
    # LLaMA-3.1-70B-shaped GQA decode: 5 of 8 KV groups, 8 query heads each
    "llama31_70b_gqa": Workload("llama31_70b_gqa", B=32, H_q=64, H_kv=8, N_kv=4096,
                                d=128, top_k=5, dtype="bf16", index="perm", seed=3000),
    # the longest context the pages evaluate (16K tokens), LLaMA-2-7B and
    # LLaMA-3.1-70B shapes
    "llama2_7b_ctx16k": Workload("llama2_7b_ctx16k", B=16, H_q=32, H_kv=32, N_kv=16384, d=128,
                                 top_k=16, dtype="fp16", index="zipf", seed=2600),
    "llama31_70b_gqa_ctx16k": Workload("llama31_70b_gqa_ctx16k", B=8, H_q=64, H_kv=8,
                                       N_kv=16384, d=128, top_k=5, dtype="bf16", index="perm",
                                       seed=3100),
}


def sweep(B, N_kv, top_k, point=0):
    """LLaMA-2-7B-shaped scaling-sweep point (H=32, d=128, fp16)."""
    return Workload(f"sweep_B{B}_N{N_kv}_k{top_k}", B=B, H_q=32, H_kv=32, N_kv=N_kv,
                    d=128, top_k=top_k, dtype="fp16", index="perm",
                    seed=4000 + point)


SWEEP_B = (1, 8, 32, 64, 128, 256)
SWEEP_N = (512, 1920, 4096, 8192)
SWEEP_TOPK = (8, 16, 24, 32)


def make_index(w: Workload):
    """int32 [B, top_k] head ids, distinct within each row, from a CPU generator."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed + 7)
    if w.index == "perm":
        rows = [torch.randperm(w.H_kv, generator=g)[: w.top_k] for _ in range(w.B)]
    elif w.index == "zipf":
        # popularity w_r = 1/r over ranks r = 1..H; ranks map to heads by one
        # seeded permutation; each row samples top_k ranks without replacement
        rank_to_head = torch.randperm(w.H_kv, generator=g)
        weights = 1.0 / torch.arange(1, w.H_kv + 1, dtype=torch.float64)
        rows = [rank_to_head[torch.multinomial(weights, w.top_k, replacement=False,
                                               generator=g)]
                for _ in range(w.B)]
    else:
        raise ValueError(f"unknown index recipe {w.index!r}")
    if w.B == 0 or w.top_k == 0:
        return torch.zeros((w.B, w.top_k), dtype=torch.int32)
    return torch.stack(rows).to(torch.int32).contiguous()


def make_tokens(w: Workload, n_sel, seed_offset=13):
    """int32 [B, top_k, n_sel] key positions for head x token sparsity: for every
    unit a uniform random subset of [0, N_kv) without repetition when n_sel <=
    N_kv (else every position once and the rest drawn again), sorted, from a
    CPU generator seeded with seed + seed_offset."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed + seed_offset)
    units = w.B * w.top_k
    if n_sel <= w.N_kv:
        keys = torch.rand((units, w.N_kv), generator=g).argsort(dim=1)[:, :n_sel]
    else:
        extra = torch.randint(0, w.N_kv, (units, n_sel - w.N_kv), generator=g)
        keys = torch.cat([torch.arange(w.N_kv).expand(units, -1), extra], dim=1)
    return keys.sort(dim=1).values.to(torch.int32).reshape(w.B, w.top_k, n_sel).contiguous()


def make_qkv(w: Workload, device="cpu"):
    """Q [B, H_q, d], K and V [B, H_kv, N_kv, d], N(0,1) rounded to the workload dtype."""
    dt = TORCH_DTYPE[w.dtype]
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    q = torch.randn((w.B, w.H_q, w.d), generator=g, device=device, dtype=torch.float32).to(dt)
    k = torch.empty((w.B, w.H_kv, w.N_kv, w.d), device=device, dtype=dt)
    v = torch.empty_like(k)
    # draw in slabs so a multi-GB cache never needs an fp32 copy of itself
    for dst in (k, v):
        flat = dst.view(-1, w.N_kv * w.d)
        for i in range(0, flat.shape[0], 256):
            rows = flat[i:i + 256]
            rows.copy_(torch.randn(rows.shape, generator=g, device=device,
                                   dtype=torch.float32))
    return q, k, v


def make_out(w: Workload, device="cpu"):
    """Output [B, H_q, d] filled with the sentinel bit pattern."""
    out = torch.empty((w.B, w.H_q, w.d), dtype=TORCH_DTYPE[w.dtype], device=device)
    out.view(torch.int16).fill_(SENTINEL[w.dtype] - (1 << 16) if SENTINEL[w.dtype] >= 1 << 15
                                else SENTINEL[w.dtype])
    return out


# ---------------------------------------------------------------- selective GEMM (MLP)

@dataclass(frozen=True)
class MlpWorkload:
    """One decoder MLP at decode time: batch B, hidden d, D = 4d neurons (OPT).
    `density` is the fraction of neurons in the union of the batch's active sets."""
    name: str
    B: int
    d: int
    D: int
    density: float
    dtype: str = "fp16"
    seed: int = 0

    def with_(self, **kw):
        return replace(self, **kw)

    def n_union(self):
        return max(1, int(round(self.density * self.D)))

    def algorithmic_bytes(self):
        """Selected rows of W1t and W2t, x read, y written, the active mask, S."""
        n = self.n_union()
        return 2 * n * self.d * 2 + 2 * self.B * self.d * 2 + self.B * self.D + 4 * self.D


MLP_CONFIGS = {
    # OPT-66B MLP (hidden 9216, 36864 neurons) at a small decode batch
    "opt66b_mlp": MlpWorkload("opt66b_mlp", B=8, d=9216, D=36864, density=0.3, dtype="fp16",
                              seed=5000),
}


def make_mlp(w: MlpWorkload, device="cpu"):
    """x [B, d] ~ N(0,1); W1t [D, d] ~ N(0, 1/d); W2t [D, d] ~ N(0, 1/n_union), so
    hidden pre-activations and outputs are O(1).  active [B, D] uint8: a seeded
    union of n_union neurons, each of which is active in at least one row (rows
    pick random subsets of the union)."""
    dt = TORCH_DTYPE[w.dtype]
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    x = torch.randn((w.B, w.d), generator=g, device=device).to(dt)
    W1t = (torch.randn((w.D, w.d), generator=g, device=device) / w.d ** 0.5).to(dt)
    W2t = (torch.randn((w.D, w.d), generator=g, device=device) / w.n_union() ** 0.5).to(dt)
    gc = torch.Generator().manual_seed(w.seed + 7)
    union = torch.randperm(w.D, generator=gc)[: w.n_union()]
    owner = torch.randint(0, w.B, (len(union),), generator=gc)
    extra = torch.rand((w.B, len(union)), generator=gc) < 0.3
    active = torch.zeros((w.B, w.D), dtype=torch.uint8)
    active[owner, union] = 1
    cols = union.unsqueeze(0).expand(w.B, -1)
    active[extra.nonzero(as_tuple=True)[0], cols[extra]] = 1
    return x, W1t, W2t, active.to(device)
