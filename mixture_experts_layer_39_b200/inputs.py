"""Seeded synthetic inputs for the MoE expert layer.

This module only draws random numbers; it holds none of the layer's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it
without sharing any code of the method.

Workloads (shapes and value distributions):

  tiny   T=512   d=256  f=512  E=8   k=4  learned-style routing
  e8     T=16384 d=2048 f=1024 E=8   k=4  learned-style routing
  e128   T=16384 d=2048 f=1024 E=128 k=4  learned-style routing
  skew   T=32768 d=2048 f=1024 E=128 k=4  router bias b_e = 2*ln(1/(e+1))
  mxfp8  T=32768 d=4096 f=1536 E=128 k=4  uniform random expert ids,
                                          drawn without replacement
  e8_shared  e8 plus one shared expert of d_ff 1024 (every token)
  mxfp8_small T=8192 d=4096 f=1536 E=32 k=4, as mxfp8 (1024 rows per expert)

Values: x ~ N(0,1); router weight, gate/up and down weights ~ N(0, 1/d);
upstream gradient dY ~ N(0,1); everything rounded to bf16 (round to
nearest even, done by torch's dtype cast).  The pages' benchmark modes
are "learned" routing (router logits from the weights) and "random
routing" used for the trillion-parameter system runs (Olmo-core 3
introduction page, key-numbers table caveats; bigchange.ai article,
section on the three numbers).  No dataset is used: these draws stand in
for the pages' training data.

Layouts (row-major):
  x      [T, d]        bf16
  w_r    [E, d]        bf16   router weight
  w_gu   [E, 2f, d]    bf16   rows 0..f-1 gate, rows f..2f-1 up
  w_d    [E, d, f]     bf16   down projection
  dy     [T, d]        bf16   upstream gradient of y
  bias   [E]           fp32 or None
  route  [T, k]        int32 or None (random-routing expert ids)
  w_gu_s [2fs, d]      bf16   shared expert gate/up (only with shared_ff = fs > 0)
  w_d_s  [d, fs]       bf16   shared expert down projection
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    f: int
    E: int
    k: int
    skew_bias: bool = False
    random_routing: bool = False
    mxfp8: bool = False
    shared_ff: int = 0

    @property
    def routed_rows(self) -> int:
        return self.T * self.k

    @property
    def max_padded_rows(self) -> int:
        # each expert segment is padded to a multiple of 32 rows
        return self.T * self.k + 31 * self.E

    def gemm_flops_fwd_bwd(self) -> float:
        # gate/up 4dfM + down 2dfM forward, twice that backward
        return 18.0 * self.d * self.f * self.T * self.k

    def shared_flops_fwd_bwd(self) -> float:
        # the same for the shared expert over all T tokens
        return 18.0 * self.d * self.shared_ff * self.T


CONFIGS = {
    "tiny": MoEConfig("tiny", 512, 256, 512, 8, 4),
    "e8": MoEConfig("e8", 16384, 2048, 1024, 8, 4),
    "e128": MoEConfig("e128", 16384, 2048, 1024, 128, 4),
    "skew": MoEConfig("skew", 32768, 2048, 1024, 128, 4, skew_bias=True),
    "mxfp8": MoEConfig("mxfp8", 32768, 4096, 1536, 128, 4,
                       random_routing=True, mxfp8=True),
    "e8_shared": MoEConfig("e8_shared", 16384, 2048, 1024, 8, 4, shared_ff=1024),
    # the mxfp8 workload's d, f and rows per expert (1024) at a quarter of its
    # tokens and experts: small enough for full profiler captures
    "mxfp8_small": MoEConfig("mxfp8_small", 8192, 4096, 1536, 32, 4,
                             random_routing=True, mxfp8=True),
}


def custom_config(T, d, f, E, k, name="custom", skew_bias=False,
                  random_routing=False, mxfp8=False, shared_ff=0) -> MoEConfig:
    return MoEConfig(name, T, d, f, E, k, skew_bias, random_routing, mxfp8, shared_ff)


def _randn(shape, std, gen, device):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def make_inputs(cfg: MoEConfig, seed: int = 0, device="cpu") -> dict:
    """Draw one step's inputs for `cfg` with a seeded torch generator.

    The generator lives on `device`, so CPU and CUDA draws differ; a test
    that compares two implementations draws once and hands the same
    tensors to both.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    std_w = 1.0 / math.sqrt(cfg.d)
    out = {
        "x": _randn((cfg.T, cfg.d), 1.0, gen, dev),
        "w_r": _randn((cfg.E, cfg.d), std_w, gen, dev),
        "w_gu": _randn((cfg.E, 2 * cfg.f, cfg.d), std_w, gen, dev),
        "w_d": _randn((cfg.E, cfg.d, cfg.f), std_w, gen, dev),
        "dy": _randn((cfg.T, cfg.d), 1.0, gen, dev),
        "bias": None,
        "route": None,
    }
    if cfg.skew_bias:
        rank = torch.arange(1, cfg.E + 1, dtype=torch.float64)
        out["bias"] = (2.0 * torch.log(1.0 / rank)).to(torch.float32).to(dev)
    if cfg.random_routing:
        noise = torch.rand((cfg.T, cfg.E), generator=gen, device=dev)
        out["route"] = noise.argsort(dim=1)[:, : cfg.k].to(torch.int32).contiguous()
    if cfg.shared_ff > 0:  # drawn last: the other tensors do not change
        out["w_gu_s"] = _randn((2 * cfg.shared_ff, cfg.d), std_w, gen, dev)
        out["w_d_s"] = _randn((cfg.d, cfg.shared_ff), std_w, gen, dev)
    return out
