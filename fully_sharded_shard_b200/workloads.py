"""Seeded synthetic workloads: parameter-group shapes and value generators.

This module only names shapes and draws random numbers.  It holds none of the
sharding step's arithmetic (no chunking, padding, casting or reduction), so
both the CUDA path and the CPU oracle can take their inputs from it.

Workload shapes follow the pages' examples:

* ``tiny_mlp`` -- Linear(16, 32) + Linear(32, 4) with biases, the two-rank
  probe model of "Sharded Training: FSDP2, DTensor, Tensor and Pipeline
  Parallelism" (ZeroRedundancyOptimizer paragraph), N = 2.
* ``llama_block`` -- one Llama-style decoder block as one group (the
  "apply fully_shard bottom-up, one group per block" rule of the fully_shard
  paragraph on the same page), N = 8.
* ``uneven`` -- embedding / LM head with 32003 rows plus 64 random shapes,
  N = 6: every parameter is padded ("padded internally when rows do not
  divide evenly", fully_shard paragraph).
* ``moe`` -- an MoE layer with 64 experts sharded per expert ("PyTorch FSDP2
  Guide: Distributed LLM Training with DTensor", section "1. Per-Parameter
  Sharding with Native DeviceMesh", irregular and MoE compatibility), N = 8.
* ``llama7b`` -- 32 Llama-2-7B-shaped blocks plus the root group (embedding,
  final norm, LM head), N = 8.  The 7B figure is the 16 bytes/param example
  of the Sharded Training page's opening paragraph.
* ``toy_llm`` -- the demo transformer of the DTensor guide's section
  "End-to-End Implementation: Sharding a Transformer with PyTorch FSDP2"
  (vocabulary 1000, hidden size 256, 4 blocks, each block its own group and
  the embedding, final norm and LM head the root's), N = 8: its SwiGLU
  projections [1364, 256] and [256, 682] do not divide into 8 row chunks of
  equal size.

Values: fp32 master parameters ~ N(0, 0.02) (tiny_mlp: U(-0.25, 0.25));
per-rank bf16 gradients ~ N(0, sigma) with sigma = 1e-3 (tiny_mlp: 1), drawn in
fp32 and rounded to bf16 by torch; each (seed, group, step, rank) has its own
generator stream.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field
from typing import List, Sequence, Tuple

import numpy as np
import torch

Shape = Tuple[int, ...]

SUM, AVG, SUM_THEN_DIV = 0, 1, 2
OP_NAMES = {SUM: "SUM", AVG: "AVG", SUM_THEN_DIV: "SUM_THEN_DIV"}

ADAMW_DEFAULTS = dict(lr=3e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


@dataclass
class Group:
    name: str
    shapes: List[Shape]
    param_names: List[str]
    # indices of parameters whose gradient is an all-zero tensor on every rank
    zero_grad: List[int] = field(default_factory=list)
    # how many times this group occurs in the model (identical shapes)
    repeat: int = 1


@dataclass
class Workload:
    name: str
    N: int
    groups: List[Group]
    op: int
    seed: int
    master_dist: str          # "normal" or "uniform"
    master_scale: float       # std for normal, half-width for uniform
    grad_sigma: float
    steps: int = 1

    def total_params(self) -> int:
        return sum(g.repeat * sum(int(np.prod(s)) for s in g.shapes)
                   for g in self.groups)


# ---------------------------------------------------------------------------
# shapes
# ---------------------------------------------------------------------------
def _block(d: int, ffn: int, kv: int, tag: str = "") -> Group:
    shapes = [(d, d), (kv, d), (kv, d), (d, d), (ffn, d), (ffn, d), (d, ffn),
              (d,), (d,)]
    names = ["wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down", "norm1", "norm2"]
    return Group("block" + tag, shapes, names)


def tiny_mlp() -> Workload:
    g = Group("root", [(32, 16), (32,), (4, 32), (4,)],
              ["0.weight", "0.bias", "2.weight", "2.bias"])
    return Workload("tiny_mlp", 2, [g], AVG, 0, "uniform", 0.25, 1.0, steps=3)


def toy_llm() -> Workload:
    """The DTensor guide's demo model, SimpleLLM(vocab_size=1000, hidden_dim=256,
    num_layers=4): per block two LayerNorms (weight and bias), the fused QKV
    projection [3 * 256, 256], the output projection [256, 256], the SwiGLU
    gate/up projection [2 * int(4 * 256 * 2 / 3), 256] = [1364, 256] and the
    down projection [256, 682], all without biases; the root group holds the
    embedding [1000, 256], the final LayerNorm and the output (LM head)
    projection [1000, 256]."""
    d, ffn, vocab = 256, int(4 * 256 * 2 / 3), 1000
    blk = Group("block", [(d,), (d,), (3 * d, d), (d, d), (d,), (d,), (2 * ffn, d), (d, ffn)],
                ["norm1.weight", "norm1.bias", "qkv_proj.weight", "out_proj.weight",
                 "norm2.weight", "norm2.bias", "mlp_gate_up.weight", "mlp_down.weight"])
    blk.repeat = 4
    root = Group("root", [(vocab, d), (d,), (d,), (vocab, d)],
                 ["tok_embeddings.weight", "norm.weight", "norm.bias", "output.weight"])
    return Workload("toy_llm", 8, [blk, root], AVG, 3, "normal", 0.02, 1e-3)


def llama_block(scale: int = 1) -> Workload:
    d, ffn, kv = 4096 // scale, 14336 // scale, 1024 // scale
    return Workload("llama_block" + ("" if scale == 1 else f"_div{scale}"), 8,
                    [_block(d, ffn, kv)], AVG, 0, "normal", 0.02, 1e-3)


def _random_shapes(rng: np.random.Generator, count: int, dmax: int,
                   widths: Sequence[int]) -> List[Shape]:
    out: List[Shape] = []
    for _ in range(count):
        d0 = int(rng.integers(1, dmax + 1))          # U{1..dmax}
        w = int(widths[int(rng.integers(0, len(widths)))])
        out.append((d0,) if w == 1 else (d0, w))
    return out


def uneven(scale: int = 1) -> Workload:
    seed = 1
    rng = np.random.default_rng(seed)
    vocab, d = 32003 // scale, 4096 // scale
    if scale == 1:
        widths, dmax = (1, 64, 4096), 5000
    else:
        widths, dmax = (1, max(2, 64 // scale), d), max(8, 5000 // scale)
    shapes: List[Shape] = [(vocab, d), (vocab, d), (d,)]
    names = ["tok_embeddings", "output", "norm"]
    rs = _random_shapes(rng, 64, dmax, widths)
    shapes += rs
    names += [f"rand{k}" for k in range(len(rs))]
    g = Group("uneven", shapes, names)
    return Workload("uneven" + ("" if scale == 1 else f"_div{scale}"), 6, [g],
                    SUM_THEN_DIV, seed, "normal", 0.02, 1e-3)


def moe(scale: int = 1, experts: int = 64, zero_experts: int = 16) -> Workload:
    d, ff = 2048 // scale, 1408 // scale
    shapes: List[Shape] = [(d, d)] * 4 + [(experts, d)]
    names = ["wq", "wk", "wv", "wo", "router"]
    for e in range(experts):
        shapes += [(ff, d), (ff, d), (d, ff)]
        names += [f"experts.{e}.gate", f"experts.{e}.up", f"experts.{e}.down"]
    rng = np.random.default_rng(0)
    unrouted = sorted(int(e) for e in rng.choice(experts, zero_experts, replace=False))
    zero = [5 + 3 * e + k for e in unrouted for k in range(3)]
    g = Group("moe", shapes, names, zero_grad=zero)
    return Workload("moe" + ("" if scale == 1 else f"_div{scale}"), 8, [g], AVG, 0,
                    "normal", 0.02, 1e-3)


def small_params(count: int = 3000, seed: int = 5) -> Workload:
    """A group of many small parameters (biases, norms, small tables): not one
    of the pages' configurations -- a measurement of the copy-outs' packed
    path, where every (rank, parameter) run is a few hundred elements.
    d0 ~ U{1..299}, width from {1, 3, 17, 64} (1 = a 1-D parameter), N = 8."""
    rng = np.random.default_rng(seed)
    shapes = _random_shapes(rng, count, 299, (1, 3, 17, 64))
    g = Group("small", shapes, [f"p{k}" for k in range(count)])
    return Workload("small_params", 8, [g], AVG, seed, "normal", 0.02, 1e-3)


def llama7b(scale: int = 1, layers: int = 32) -> Workload:
    d, ffn, vocab = 4096 // scale, 11008 // scale, 32000 // scale
    blk = _block(d, ffn, d)
    blk.repeat = layers
    root = Group("root", [(vocab, d), (d,), (vocab, d)],
                 ["tok_embeddings", "norm", "output"])
    return Workload("llama7b" + ("" if scale == 1 else f"_div{scale}"), 8,
                    [blk, root], AVG, 0, "normal", 0.02, 1e-3)


def by_name(name: str) -> Workload:
    """A workload by name; ``<name>_div<k>`` divides its dims by k and
    ``llama7b..._l<L>`` keeps L blocks (small cases for profiling)."""
    import re
    table = {
        "tiny_mlp": tiny_mlp,
        "llama_block": llama_block,
        "uneven": uneven,
        "moe": moe,
        "llama7b": llama7b,
        "small_params": small_params,
        "toy_llm": toy_llm,
    }
    if name in table:
        return table[name]()
    m = re.fullmatch(r"(llama_block|uneven|moe|llama7b)(?:_div(\d+))?(?:_l(\d+))?", name)
    if not m:
        raise KeyError(name)
    base, div, layers = m.group(1), int(m.group(2) or 1), m.group(3)
    if base == "llama7b":
        wl = llama7b(div, layers=int(layers)) if layers else llama7b(div)
    else:
        if layers:
            raise KeyError(name)
        wl = table[base](div) if div != 1 else table[base]()
    wl.name = name
    return wl


# ---------------------------------------------------------------------------
# values
# ---------------------------------------------------------------------------
def stream_seed(*parts) -> int:
    """A 63-bit seed derived from the parts (stable across runs/platforms)."""
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(stream_seed(*parts))
    return g


def fill_master(t: torch.Tensor, wl: Workload, *parts) -> torch.Tensor:
    """Fill an fp32 tensor (the full-parameter arena) with the master values."""
    g = generator(t.device, wl.seed, "master", *parts)
    if wl.master_dist == "uniform":
        t.uniform_(-wl.master_scale, wl.master_scale, generator=g)
    else:
        t.normal_(0.0, wl.master_scale, generator=g)
    return t


def fill_grads_bf16(t: torch.Tensor, wl: Workload, *parts, chunk: int = 1 << 26) -> torch.Tensor:
    """Fill a bf16 tensor with N(0, grad_sigma) values drawn in fp32 and
    rounded to bf16 by torch (RNE).  Drawn in chunks to bound the fp32 temp."""
    assert t.dtype == torch.bfloat16
    flat = t.view(-1)
    g = generator(t.device, wl.seed, "grad", *parts)
    for lo in range(0, flat.numel(), chunk):
        hi = min(flat.numel(), lo + chunk)
        tmp = torch.empty(hi - lo, dtype=torch.float32, device=t.device)
        tmp.normal_(0.0, wl.grad_sigma, generator=g)
        flat[lo:hi].copy_(tmp)
    return t


def zero_param_ranges(t_rank: torch.Tensor, arena_off: Sequence[int],
                      numels: Sequence[int], which: Sequence[int]) -> None:
    """Write an all-zero gradient for parameters ``which`` (an unrouted
    expert's gradient tensor) into one rank's gradient arena."""
    for i in which:
        a = int(arena_off[i])
        t_rank[a:a + int(numels[i])].zero_()
