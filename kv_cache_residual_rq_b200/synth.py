"""Seeded synthetic workloads (inputs only; none of the method's arithmetic).

The pages measure ResidualQuant on looped language models (Ouro, Huginn)
with mathematical-reasoning and code benchmarks; neither models nor
benchmarks are available, so these generators stand in for the KV caches
such models write.  Shapes follow the five workloads of the build (an
Ouro-1.4B-like stack: 4 loops, 24 layers, 16 heads, head_dim 128).

Recipe, per (workload, layer, tensor):
  a_c    = exp(0.5 * N(0,1)) per (kv head, channel)        (channel outliers)
  ref    = bf16(N(0,1) * a_c)                              (final loop, BF16)
  loop l = bf16(f32(ref) + sigma_l * N(0,1))               (non-final loops)
  q      = bf16(N(0,1))
with torch's Philox generator seeded from (workload seed, layer, tensor).
Both the CUDA path and the oracle receive exactly these tensors (the oracle
gets host copies).
"""
import dataclasses
import math
from typing import List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    loops: int                 # L; loop L is the BF16 reference
    layers: int
    batch: int
    ctx: int
    q_heads: int
    kv_heads: int
    head_dim: int
    group: int
    bits: tuple                # bits of loops 1 .. L-1
    sigma: tuple               # residual sigma of loops 1 .. L-1
    seed: int

    @property
    def G(self):
        return self.q_heads // self.kv_heads


def _sigma_linear(loops):
    # loop l = ref + 0.1 * (L - l) * N(0,1)
    return tuple(0.1 * (loops - l) for l in range(1, loops))


def _sigma_geometric(loops, hi, lo):
    n = loops - 1
    return tuple(hi * (lo / hi) ** ((l - 1) / (n - 1)) for l in range(1, loops))


TINY = Workload("tiny", 4, 1, 1, 256, 8, 2, 64, 32, (2, 2, 2), _sigma_linear(4), 0)
OURO = Workload("ouro1.4b_decode", 4, 24, 16, 4096, 16, 16, 128, 32, (2, 2, 2),
                (0.15, 0.10, 0.05), 1)
MIXED = Workload("mixed_precision_32k", 4, 24, 8, 32768, 16, 16, 128, 32, (4, 2, 2),
                 _sigma_linear(4), 2)
DEEP = Workload("deep_loop_gqa", 8, 16, 32, 8192, 32, 8, 128, 64, (2,) * 7,
                _sigma_geometric(8, 0.3, 0.02), 3)
ENCODE = Workload("encode_prefill_32k", 4, 24, 1, 32768, 16, 16, 128, 32, (2, 2, 2),
                  _sigma_linear(4), 4)

WORKLOADS = [TINY, OURO, MIXED, DEEP, ENCODE]
BY_NAME = {w.name: w for w in WORKLOADS}

# batch sweep of the encode workload: decode at ctx 32768 under a KV budget
SWEEP_BATCHES = (1, 2, 4, 8, 12, 16, 32, 64)
KV_BUDGET_BYTES = 120e9


def _gen(w: Workload, layer: int, tensor: int, device):
    g = torch.Generator(device=device)
    g.manual_seed(w.seed * 1_000_003 + layer * 16 + tensor)
    return g


def channel_scales(w: Workload, layer: int, kind: int, device="cuda"):
    """a_c for kind 0 (K) or 1 (V): [Hkv, 1, d] fp32."""
    g = _gen(w, layer, 8 + kind, device)
    z = torch.randn((w.kv_heads, 1, w.head_dim), generator=g, device=device)
    return torch.exp(0.5 * z)


def reference(w: Workload, layer: int, kind: int, device="cuda", batch=None, ctx=None):
    """Final-loop K (kind 0) or V (kind 1): bf16 [B, Hkv, T, d]."""
    b = w.batch if batch is None else batch
    t = w.ctx if ctx is None else ctx
    g = _gen(w, layer, kind, device)
    a = channel_scales(w, layer, kind, device)
    x = torch.randn((b, w.kv_heads, t, w.head_dim), generator=g, device=device)
    return (x * a).to(torch.bfloat16)


def loop_kv(w: Workload, layer: int, kind: int, loop: int, ref: torch.Tensor):
    """Non-final loop `loop` (1-based) of K/V: bf16(f32(ref) + sigma * N(0,1))."""
    g = _gen(w, layer, 2 + 2 * loop + kind, ref.device)
    noise = torch.randn(ref.shape, generator=g, device=ref.device)
    return (ref.float() + w.sigma[loop - 1] * noise).to(torch.bfloat16)


def query(w: Workload, layer: int, loop: int, device="cuda", batch=None, step=0):
    """Decode query of (layer, loop): bf16 [B, Hq, d]."""
    b = w.batch if batch is None else batch
    g = torch.Generator(device=device)
    g.manual_seed(w.seed * 7_000_003 + step * 100_003 + layer * 64 + loop)
    return torch.randn((b, w.q_heads, w.head_dim), generator=g, device=device).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """Host numpy uint16 view of a bf16 tensor (for the oracle)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def storage_bits_per_element(w: Workload):
    """Stored bits per (token, kv head, channel), summed over all loops."""
    total = 16.0                                   # the reference loop
    for b in w.bits:
        total += 16.0 if b == 16 else b + 16.0 / w.group
    return total


def kv_bytes_per_sequence(w: Workload, ctx: int, quantized: bool):
    """KV bytes of one sequence across all layers and loops."""
    per_elem = storage_bits_per_element(w) / 8 if quantized else 2.0 * w.loops
    return int(2 * w.layers * w.kv_heads * ctx * w.head_dim * per_elem)
