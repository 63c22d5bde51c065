"""Seeded synthetic workloads for the NVFP4 W4A4 routed-MoE feed-forward layer.

This module only draws random inputs.  It holds none of the layer's arithmetic (no
quantisation, routing or GEMM), so both the CUDA path and the CPU oracle can be fed from
it.  Draws use torch's seeded generators: on the CPU for sizes the oracle checks
directly, on the GPU (Philox) for the full-size workloads, whose sampled parts the tests
copy back to the host.

Shapes follow the routed-expert layer of the pages: 512 routed experts (Eider, "Qwen3.8
Flash Next"), prefill chunks of up to 512 tokens (Eider, "Performance"), 16 decode rows
(DwarfStar CUDA multi-GPU doc), and a dense NVFP4 MLP (Eider, "Qwen3.8 27B").
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens (rows)
    H: int          # hidden size
    I: int          # expert intermediate size
    E: int          # experts
    k: int          # experts per token
    zipf_s: float = 0.0        # >0: skew router logits by a Zipf(s) popularity bias
    outlier_frac: float = 0.0  # fraction of hidden channels scaled by outlier_gain
    outlier_gain: float = 1.0
    dense: bool = False        # single expert, no routing (E=1, k=1, w=1)

    @property
    def pairs(self) -> int:
        return self.T * self.k


WORKLOADS = {
    # tiny routed layer: T8 H256 I128 E8 top-2
    "tiny": Workload("tiny", T=8, H=256, I=128, E=8, k=2),
    # decode-shaped routed layer: 16 rows, 512 experts, top-10
    "decode": Workload("decode", T=16, H=2048, I=512, E=512, k=10),
    # prefill chunk: 512 tokens, Zipf(1.1)-skewed experts, 1% outlier channels x20
    "prefill_chunk": Workload("prefill_chunk", T=512, H=2048, I=512, E=512, k=10,
                              zipf_s=1.1, outlier_frac=0.01, outlier_gain=20.0),
    # long prefill: 4096 tokens, 256 experts, top-8
    "long_prefill": Workload("long_prefill", T=4096, H=4096, I=1024, E=256, k=8),
    # dense NVFP4 W4A4 MLP (one expert, no routing), 512 rows and 1 row
    "dense": Workload("dense", T=512, H=5120, I=17408, E=1, k=1, dense=True),
    "dense_t1": Workload("dense_t1", T=1, H=5120, I=17408, E=1, k=1, dense=True),
}


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some sizes changed (reduced parity cases)."""
    return dataclasses.replace(w, **changes)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_activations(w: Workload, seed: int = 0, device="cpu") -> dict:
    """x bf16 [T, H] and router logits fp32 [T, E].

    x ~ N(0, 1), with a seeded set of floor(outlier_frac*H) channels multiplied by
    outlier_gain before the (round-to-nearest-even) bf16 conversion.  Logits ~ N(0, 1),
    plus, when zipf_s > 0, bias_e = ln p_e with p_e proportional to rank_e^-s over a seeded
    random ranking of the experts.  Dense workloads get all-zero [T, 1] logits.
    """
    g = _gen(seed, device)
    x = torch.randn(w.T, w.H, generator=g, device=device, dtype=torch.float32)
    if w.outlier_frac > 0:
        n_out = int(math.floor(w.outlier_frac * w.H))
        gc = _gen(seed + 101, "cpu")
        ch = torch.randperm(w.H, generator=gc)[:n_out].to(device)
        x[:, ch] *= w.outlier_gain
    x = x.to(torch.bfloat16)
    if w.dense:
        logits = torch.zeros(w.T, 1, device=device, dtype=torch.float32)
    else:
        logits = torch.randn(w.T, w.E, generator=g, device=device, dtype=torch.float32)
        if w.zipf_s > 0:
            gc = _gen(seed + 202, "cpu")
            rank = torch.randperm(w.E, generator=gc).to(torch.float64) + 1.0
            p = rank.pow(-w.zipf_s)
            p = p / p.sum()
            bias = torch.log(p).to(torch.float32).to(device)
            logits = logits + bias[None, :]
    return {"x": x.contiguous(), "logits": logits.contiguous()}


def make_weights(w: Workload, seed: int = 0, device="cpu") -> dict:
    """fp32 expert weights: w_gate, w_up [E, I, H] and w_down [E, H, I], each drawn
    N(0, sigma = 1/sqrt(fan_in)) with fan_in = H for gate/up and I for down."""
    g = _gen(seed + 1, device)
    sg = 1.0 / math.sqrt(w.H)
    sd = 1.0 / math.sqrt(w.I)
    w_gate = torch.randn(w.E, w.I, w.H, generator=g, device=device, dtype=torch.float32) * sg
    w_up = torch.randn(w.E, w.I, w.H, generator=g, device=device, dtype=torch.float32) * sg
    w_down = torch.randn(w.E, w.H, w.I, generator=g, device=device, dtype=torch.float32) * sd
    return {"w_gate": w_gate, "w_up": w_up, "w_down": w_down}


def make_expert_weights(w: Workload, e: int, seed: int = 0, device="cpu") -> dict:
    """fp32 weights of expert e alone, same distributions as make_weights, drawn from a
    generator of their own (seeded by seed and e).  For CPU-side consumers that need a few
    experts of a large layer without drawing all of them: the values differ from
    make_weights' draw of the same expert."""
    g = _gen(1_000_003 * (seed + 1) + e, device)
    sg = 1.0 / math.sqrt(w.H)
    sd = 1.0 / math.sqrt(w.I)
    w_gate = torch.randn(w.I, w.H, generator=g, device=device, dtype=torch.float32) * sg
    w_up = torch.randn(w.I, w.H, generator=g, device=device, dtype=torch.float32) * sg
    w_down = torch.randn(w.H, w.I, generator=g, device=device, dtype=torch.float32) * sd
    return {"w_gate": w_gate, "w_up": w_up, "w_down": w_down}
