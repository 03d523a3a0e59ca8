"""Seeded synthetic inputs for branch attention.

This module only draws random numbers and packs them into the shapes of the
workloads on the pages (EAGLE-3 training-time-test branches and DFlash-style
block drafts over packed, variable-length sequences). It holds none of the
method's arithmetic, so both the fp64 oracle tests and the CUDA path can take
their inputs from here without sharing any attention code.

Draw order per problem (one seed, ``1000 + config index``):

1. document lengths and anchors, on a CPU ``torch.Generator``;
2. q, k, v, then qb, kb, vb, then dO (main) and dO (branch), on a generator of
   the target device seeded with the same seed.  CPU and CUDA generators give
   different streams, so a problem is identified by (config, seed, device).

All tensors are bf16 draws of N(0, 1).  Layouts (row-major, last dim
contiguous):

* ``q``  [S, Hq, d],   ``k``/``v``   [S, Hkv, d]
* ``qb`` [Nb, B, Hq, d], ``kb``/``vb`` [Nb, B, Hkv, d]
* ``do`` like ``q``, ``dob`` like ``qb``
* ``cu_seqlens`` int32 [ndoc + 1], ``anchors`` int32 [Nb] (ascending)
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

CHAIN = 0  # EAGLE-3 training-time test: depth t sees branch keys u <= t
BLOCK = 1  # DFlash-style block draft: all B keys of its own block


@dataclass(frozen=True)
class Config:
    name: str
    S: int
    ndoc: int
    lengths: str  # "single" | "dirichlet" | "lognormal"
    Hq: int
    Hkv: int
    d: int
    anchors: str  # "uniform" (sample n without replacement) | "every"
    n_anchors: int
    B: int
    mode: int
    R: int
    backward: bool
    description: str = ""


CONFIGS = [
    Config("tiny_fwd", 256, 1, "single", 4, 4, 64, "uniform", 8, 4, CHAIN, 2, False,
           "1 document S=256, H=4, d=64; 8 depth-4 chain branches; R=2; forward only"),
    Config("eagle3_8k", 8192, 4, "dirichlet", 32, 8, 128, "every", 8192, 3, CHAIN, 4, True,
           "packed S=8192 from 4 Dirichlet documents; GQA 32/8, d=128; depth-3 chain "
           "branch at every position; R=4"),
    Config("dflash_32k", 32768, 8, "dirichlet", 32, 8, 128, "uniform", 1024, 16, BLOCK, 8, True,
           "packed S=32768 from 8 documents; GQA 32/8, d=128; 1024 anchors; 16-token "
           "bidirectional blocks; R=8"),
    Config("eagle3_64k", 65536, 16, "lognormal", 32, 8, 128, "every", 65536, 3, CHAIN, 8, True,
           "packed S=65536 from 16 log-normal documents (mean 4096); GQA 32/8, d=128; "
           "depth-3 chain branch at every position; R=8"),
    Config("eagle3_256k", 262144, 1, "single", 32, 8, 128, "every", 262144, 3, CHAIN, 8, True,
           "one document S=262144; GQA 32/8, d=128; depth-3 chain branch at every "
           "position; R=8"),
]

CONFIG_BY_NAME = {c.name: c for c in CONFIGS}


def seed_of(cfg_index: int) -> int:
    return 1000 + cfg_index


def _lengths(cfg: Config, g: torch.Generator) -> list[int]:
    S, n = cfg.S, cfg.ndoc
    if cfg.lengths == "single":
        assert n == 1
        return [S]
    if cfg.lengths == "dirichlet":
        # Dirichlet(1) = normalised i.i.d. Exp(1) draws.
        e = torch.empty(n, dtype=torch.float64).exponential_(1.0, generator=g)
        w = (e / e.sum()).tolist()
        out = [max(1, int(math.floor(S * wi))) for wi in w[:-1]]
        out.append(S - sum(out))
        assert out[-1] >= 1
        return out
    if cfg.lengths == "lognormal":
        sigma = 0.5
        mu = math.log(S / n) - sigma * sigma / 2.0
        z = torch.randn(n, dtype=torch.float64, generator=g)
        x = torch.exp(mu + sigma * z)
        share = (x / x.sum() * S).tolist()
        base = [max(1, int(math.floor(s))) for s in share]
        rem = S - sum(base)
        # largest remainder; a negative remainder (from the minimum of 1)
        # is taken from the longest documents
        order = sorted(range(n), key=lambda i: share[i] - math.floor(share[i]), reverse=True)
        i = 0
        while rem > 0:
            base[order[i % n]] += 1
            rem -= 1
            i += 1
        while rem < 0:
            j = max(range(n), key=lambda t: base[t])
            base[j] -= 1
            rem += 1
        return base
    raise ValueError(cfg.lengths)


def _anchors(cfg: Config, g: torch.Generator) -> list[int]:
    if cfg.anchors == "every":
        assert cfg.n_anchors == cfg.S
        return list(range(cfg.S))
    if cfg.anchors == "uniform":
        perm = torch.randperm(cfg.S, generator=g)[: cfg.n_anchors]
        return sorted(perm.tolist())
    raise ValueError(cfg.anchors)


@dataclass
class Problem:
    cfg: Config
    seed: int
    cu_seqlens: torch.Tensor  # int32 [ndoc+1], CPU
    anchors: torch.Tensor     # int32 [Nb], CPU
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    qb: torch.Tensor
    kb: torch.Tensor
    vb: torch.Tensor
    do: torch.Tensor | None = None
    dob: torch.Tensor | None = None
    extra: dict = field(default_factory=dict)

    @property
    def S(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def Nb(self) -> int:
        return int(self.anchors.numel())


def _randn_bf16(shape, g, device) -> torch.Tensor:
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def make_custom(lengths, anchors, *, Hq, Hkv, d, B, mode, seed, device="cpu",
                with_grad_inputs=True, cfg_name="custom", R=1) -> Problem:
    """Problem with explicit document lengths and anchors (tests, small cases)."""
    lengths = [int(x) for x in lengths]
    S = sum(lengths)
    cu = torch.tensor([0] + list(_cumsum(lengths)), dtype=torch.int32)
    anc = torch.tensor(sorted(int(a) for a in anchors), dtype=torch.int32)
    cfg = Config(cfg_name, S, len(lengths), "custom", Hq, Hkv, d, "custom", int(anc.numel()),
                 B, mode, R, with_grad_inputs)
    return _draw(cfg, seed, cu, anc, device, with_grad_inputs)


def _cumsum(xs):
    t = 0
    for x in xs:
        t += x
        yield t


def _draw(cfg, seed, cu, anc, device, with_grad_inputs) -> Problem:
    S, Nb, B = int(cu[-1]), int(anc.numel()), cfg.B
    if device == "cpu" or (isinstance(device, torch.device) and device.type == "cpu"):
        gd = torch.Generator()
    else:
        gd = torch.Generator(device=device)
    gd.manual_seed(seed)
    q = _randn_bf16((S, cfg.Hq, cfg.d), gd, device)
    k = _randn_bf16((S, cfg.Hkv, cfg.d), gd, device)
    v = _randn_bf16((S, cfg.Hkv, cfg.d), gd, device)
    qb = _randn_bf16((Nb, B, cfg.Hq, cfg.d), gd, device)
    kb = _randn_bf16((Nb, B, cfg.Hkv, cfg.d), gd, device)
    vb = _randn_bf16((Nb, B, cfg.Hkv, cfg.d), gd, device)
    do = dob = None
    if with_grad_inputs:
        do = _randn_bf16((S, cfg.Hq, cfg.d), gd, device)
        dob = _randn_bf16((Nb, B, cfg.Hq, cfg.d), gd, device)
    return Problem(cfg, seed, cu, anc, q, k, v, qb, kb, vb, do, dob)


def make_problem(cfg_index: int, device="cpu", with_grad_inputs=None) -> Problem:
    """The seeded problem of one of the five workload configurations."""
    cfg = CONFIGS[cfg_index]
    seed = seed_of(cfg_index)
    g = torch.Generator()
    g.manual_seed(seed)
    lengths = _lengths(cfg, g)
    anchors = _anchors(cfg, g)
    cu = torch.tensor([0] + list(_cumsum(lengths)), dtype=torch.int32)
    anc = torch.tensor(anchors, dtype=torch.int32)
    if with_grad_inputs is None:
        with_grad_inputs = cfg.backward
    return _draw(cfg, seed, cu, anc, device, with_grad_inputs)


def make_layout(cfg_index: int):
    """Only the (cu_seqlens, anchors) of a configuration: cheap, no tensors."""
    cfg = CONFIGS[cfg_index]
    g = torch.Generator()
    g.manual_seed(seed_of(cfg_index))
    lengths = _lengths(cfg, g)
    anchors = _anchors(cfg, g)
    cu = torch.tensor([0] + list(_cumsum(lengths)), dtype=torch.int32)
    return cu, torch.tensor(anchors, dtype=torch.int32)


def random_packing(S: int, ndoc: int, n_anchors: int, g: torch.Generator):
    """Random small packing for property tests: ndoc >= 1 documents of random
    positive lengths summing to S, and n_anchors distinct sorted anchors."""
    assert 1 <= ndoc <= S
    cuts = sorted(torch.randperm(S - 1, generator=g)[: ndoc - 1].add(1).tolist()) if ndoc > 1 else []
    edges = [0] + cuts + [S]
    lengths = [edges[i + 1] - edges[i] for i in range(ndoc)]
    anchors = sorted(torch.randperm(S, generator=g)[:n_anchors].tolist())
    return lengths, anchors


def sample_rows(problem_cu: torch.Tensor, anchors: torch.Tensor, B: int, n_rows: int, seed: int,
                extra=()):
    """Seeded, stratified sample of query rows (indices into the concatenated
    [main; branch] row order): about half main rows and half branch rows, always
    including the first and last row of every document, the main rows listed in
    ``extra`` (callers pass e.g. split edges), and the branch rows of anchors
    that sit at document ends."""
    g = torch.Generator()
    g.manual_seed(seed)
    cu = problem_cu.tolist()
    S = cu[-1]
    Nb = int(anchors.numel())
    must = set(int(x) for x in extra if 0 <= int(x) < S)
    ends = set()
    for i in range(len(cu) - 1):
        s, e = cu[i], cu[i + 1]
        must.add(s)
        must.add(e - 1)
        ends.add(e - 1)
    anc = anchors.tolist()
    for b, a in enumerate(anc):
        if a in ends:
            for t in range(B):
                must.add(S + b * B + t)
    n_main = min(S, n_rows // 2) if Nb else min(S, n_rows)
    n_br = min(Nb * B, n_rows - n_main)
    main = torch.randperm(S, generator=g)[:n_main].tolist()
    br = (torch.randperm(Nb * B, generator=g)[:n_br] + S).tolist() if Nb else []
    rows = sorted(must.union(main).union(br))
    return torch.tensor(rows, dtype=torch.int64)
