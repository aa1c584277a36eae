"""Seeded synthetic workloads: parameter layouts, initial params, gradients.

This module holds none of the optimizer's arithmetic.  It only draws inputs,
and both the CUDA path and the CPU oracle take the same drawn tensors.

Layouts follow the model shapes named for the FP8-moment experiments in
"Scaling FP8 training to trillion-token LLMs" (a Llama2-100M model for the
Fig. 5 moment-format ablation, a Llama2-style 7B model for the headline run):

* ``single_1m``   one tensor of 1,048,576 params; g = s*z with z ~ N(0,1) and
                  a per-element s = 10^U(-6,-1).
* ``llama2_100m`` d_model 768, 12 layers, SwiGLU FFN 2048 (w1, w2, w3), 12
                  heads, vocab 32000, tied embedding, RMSNorm gains: 110
                  tensors, 109,529,856 params.
* ``llama2_7b``   d_model 4096, 32 layers, SwiGLU FFN 11008, vocab 32000,
                  untied embedding / LM head: 291 tensors, 6,738,415,616
                  params.
* ``stress_20k``  20,000 tensors of 4,096 params (grads N(0, 1e-4)) plus 8
                  tensors of 2^28 params (heavy-tailed grads as below).
* ``pair_2x256m`` two tensors of 2^28 params (heavy-tailed grads): 7.5 GB of
                  step traffic, 4.3 GB resident -- a launch large enough for
                  DRAM counters to mean what they mean on the 7B layout, small
                  enough for a profiler capture.

Heavy-tailed gradients (llama layouts and the 2^28 tensors): per tensor a
sigma_t = 10^U(-5,-2) drawn once per run; each step g ~ N(0, sigma_t) and a
fresh 0.1% of the elements (uniform) scaled by 100.  Params start N(0, 0.02);
RMSNorm gains start at 1.0 (the Llama convention).  Every draw is seeded:
params with 1000*cfg, step k's gradients with 1000*cfg + k.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

# workload id -> the number used in the seeds
CFG_ID = {"single_1m": 1, "llama2_100m": 2, "llama2_7b": 3, "ablation_100m": 4,
          "stress_20k": 5, "pair_2x256m": 6}

ALIGN_ELEMS = 64  # tensor offsets inside flat buffers: 256 B of fp32, 64 B of codes


@dataclasses.dataclass(frozen=True)
class TensorSpec:
    name: str
    numel: int
    kind: str  # "matrix", "norm", "small", "big", "single"


def _llama(d: int, layers: int, ffn: int, vocab: int, tied: bool) -> List[TensorSpec]:
    specs = [TensorSpec("embed", vocab * d, "matrix")]
    for i in range(layers):
        for w in ("q", "k", "v", "o"):
            specs.append(TensorSpec(f"l{i}.{w}", d * d, "matrix"))
        specs.append(TensorSpec(f"l{i}.w1", d * ffn, "matrix"))
        specs.append(TensorSpec(f"l{i}.w3", d * ffn, "matrix"))
        specs.append(TensorSpec(f"l{i}.w2", ffn * d, "matrix"))
        specs.append(TensorSpec(f"l{i}.attn_norm", d, "norm"))
        specs.append(TensorSpec(f"l{i}.ffn_norm", d, "norm"))
    specs.append(TensorSpec("final_norm", d, "norm"))
    if not tied:
        specs.append(TensorSpec("lm_head", vocab * d, "matrix"))
    return specs


def layout(name: str) -> List[TensorSpec]:
    if name == "single_1m":
        return [TensorSpec("w", 1 << 20, "single")]
    if name in ("llama2_100m", "ablation_100m"):
        return _llama(768, 12, 2048, 32000, tied=True)
    if name == "llama2_7b":
        return _llama(4096, 32, 11008, 32000, tied=False)
    if name == "stress_20k":
        return ([TensorSpec(f"s{i}", 4096, "small") for i in range(20000)]
                + [TensorSpec(f"b{i}", 1 << 28, "big") for i in range(8)])
    if name == "pair_2x256m":
        return [TensorSpec(f"b{i}", 1 << 28, "big") for i in range(2)]
    raise KeyError(name)


def custom_layout(numels: List[int]) -> List[TensorSpec]:
    """Layout of arbitrary sizes with heavy-tailed grads (edge-case tests)."""
    return [TensorSpec(f"t{i}", int(n), "matrix") for i, n in enumerate(numels)]


def total_params(specs: List[TensorSpec]) -> int:
    return sum(s.numel for s in specs)


def offsets(specs: List[TensorSpec], align: int = ALIGN_ELEMS) -> List[int]:
    """Element offsets of each tensor in a flat buffer, each aligned to
    ``align`` elements."""
    out, off = [], 0
    for s in specs:
        out.append(off)
        off += (s.numel + align - 1) // align * align
    out.append(off)  # padded total
    return out


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def tensor_sigmas(specs: List[TensorSpec], cfg_id: int) -> List[float]:
    """Per-tensor gradient sigma_t = 10^U(-5,-2), drawn once per run (CPU)."""
    gen = _gen(1000 * cfg_id + 999_999, "cpu")
    u = torch.rand(len(specs), generator=gen, dtype=torch.float64)
    return [float(10.0 ** (-5.0 + 3.0 * x)) for x in u.tolist()]


def init_params_into(specs: List[TensorSpec], views: List[torch.Tensor], cfg_id: int) -> None:
    """Fill fp32 param views: N(0, 0.02), RMSNorm gains 1.0."""
    dev = views[0].device if views else "cpu"
    gen = _gen(1000 * cfg_id, dev)
    for s, v in zip(specs, views):
        if s.numel == 0:
            continue
        if s.kind == "norm":
            v.fill_(1.0)
        else:
            v.copy_(torch.randn(s.numel, generator=gen, device=dev, dtype=torch.float32) * 0.02)


def grads_into(specs: List[TensorSpec], views: List[torch.Tensor], cfg_id: int, step: int,
               sigmas: Optional[List[float]] = None) -> None:
    """Fill bf16 gradient views with step ``step``'s seeded draw."""
    dev = views[0].device if views else "cpu"
    gen = _gen(1000 * cfg_id + step, dev)
    if sigmas is None:
        sigmas = tensor_sigmas(specs, cfg_id)
    for s, v, sig in zip(specs, views, sigmas):
        n = s.numel
        if n == 0:
            continue
        if s.kind == "single":
            u = torch.rand(n, generator=gen, device=dev, dtype=torch.float32)
            z = torch.randn(n, generator=gen, device=dev, dtype=torch.float32)
            g = torch.pow(10.0, u * 5.0 - 6.0) * z
        elif s.kind == "small":
            g = torch.randn(n, generator=gen, device=dev, dtype=torch.float32) * 1e-4
        else:
            g = torch.randn(n, generator=gen, device=dev, dtype=torch.float32) * sig
            out = torch.rand(n, generator=gen, device=dev, dtype=torch.float32) < 1e-3
            g = torch.where(out, g * 100.0, g)
        v.copy_(g.to(torch.bfloat16))


class FlatModel:
    """Flat, aligned buffers holding one workload's optimizer state.

    p: fp32, g: bf16, m/v: uint8 codes (or fp32 for the fp32-moment mode);
    scale_*: fp32 [T] (init 1.0), amax_*: fp32 [T] (init 0.0).  Each tensor
    is a view at an aligned offset.
    """

    def __init__(self, specs: List[TensorSpec], device, m_fp32: bool = False,
                 v_fp32: bool = False, align: int = ALIGN_ELEMS):
        self.specs = specs
        self.device = torch.device(device)
        self.off = offsets(specs, align)
        total = self.off[-1]
        self.T = len(specs)
        self.p = torch.zeros(total, dtype=torch.float32, device=device)
        self.g = torch.zeros(total, dtype=torch.bfloat16, device=device)
        self.m = torch.zeros(total, dtype=torch.float32 if m_fp32 else torch.uint8, device=device)
        self.v = torch.zeros(total, dtype=torch.float32 if v_fp32 else torch.uint8, device=device)
        self.scale_m = torch.ones(self.T, dtype=torch.float32, device=device)
        self.scale_v = torch.ones(self.T, dtype=torch.float32, device=device)
        self.amax_m = torch.zeros(self.T, dtype=torch.float32, device=device)
        self.amax_v = torch.zeros(self.T, dtype=torch.float32, device=device)

    def view(self, buf: torch.Tensor, i: int) -> torch.Tensor:
        o = self.off[i]
        return buf[o:o + self.specs[i].numel]

    def views(self, buf: torch.Tensor) -> List[torch.Tensor]:
        return [self.view(buf, i) for i in range(self.T)]

    def bytes_resident(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.p, self.g, self.m, self.v))


HPARAMS = dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)

STEPS = {"single_1m": 10, "llama2_100m": 100, "llama2_7b": 20, "ablation_100m": 200,
         "stress_20k": 50, "pair_2x256m": 20}
