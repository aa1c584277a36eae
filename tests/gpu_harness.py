"""Runs a workload through the CUDA path (C ABI via FP8AdamW) next to the CPU
oracle on the same seeded inputs, free-running from the same initial state.

Nothing computed by the CUDA path is ever fed to the oracle: both sides start
from the seeded params and read the same seeded gradients each step.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Optional, Sequence

import numpy as np
import torch

import oracle
import pins
from fp8_quantized_adam_b200 import FP8AdamW, workloads

HP = workloads.HPARAMS
THREADS = max(1, len(os.sched_getaffinity(0)))


def bf16_host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


class Run:
    def __init__(self, specs, cfg_id: int, m_fmt: int = oracle.E4M3, v_fmt: int = oracle.E5M2,
                 subset: Optional[Sequence[int]] = None, stats: bool = False,
                 jit_every_step: bool = False, hp: Optional[dict] = None,
                 model: Optional[workloads.FlatModel] = None, init: bool = True, host: bool = False):
        self.specs, self.cfg_id = specs, cfg_id
        self.m_fmt, self.v_fmt = m_fmt, v_fmt
        self.hp = dict(HP if hp is None else hp)
        self.flags = oracle.FLAG_JIT_EVERY_STEP if jit_every_step else 0
        dev = torch.device("cuda:0")
        self.model = model or workloads.FlatModel(specs, dev, m_fp32=m_fmt == oracle.FP32,
                                                   v_fp32=v_fmt == oracle.FP32)
        M = self.model
        if init:
            workloads.init_params_into(specs, M.views(M.p), cfg_id)
        self.sigmas = workloads.tensor_sigmas(specs, cfg_id)
        self.opt = FP8AdamW(M.views(M.p), M.views(M.g), m_fmt=m_fmt, v_fmt=v_fmt, m=M.views(M.m),
                            v=M.views(M.v), scale_m=M.scale_m, scale_v=M.scale_v, amax_m=M.amax_m,
                            amax_v=M.amax_v, stats=stats, jit_every_step=jit_every_step,
                            lr=self.hp["lr"], betas=(self.hp["beta1"], self.hp["beta2"]),
                            eps=self.hp["eps"], weight_decay=self.hp["weight_decay"])
        self.subset = list(range(len(specs))) if subset is None else list(subset)
        # host mode: gradients reach the library from pinned host memory
        # through fp8adam_step_host; the device buffer is zeroed first, so
        # only the library's own copy can supply them
        self.host = host
        if host:
            self.g_host = torch.empty(M.g.numel(), dtype=torch.bfloat16, pin_memory=True)
            self.amax_host = torch.zeros(2 * len(specs), dtype=torch.float32, pin_memory=True)
        torch.cuda.synchronize()
        self.ref: Dict[int, oracle.TensorState] = {
            i: oracle.TensorState(M.view(M.p, i).cpu().numpy(), m_fmt, v_fmt) for i in self.subset}
        self.t = 0

    def draw_grads(self, t: int) -> None:
        M = self.model
        workloads.grads_into(self.specs, M.views(M.g), self.cfg_id, t, self.sigmas)

    def step(self, with_oracle: bool = True) -> None:
        self.t += 1
        self.draw_grads(self.t)
        if self.host:
            M = self.model
            self.g_host.copy_(M.g)
            M.g.zero_()
            views = [self.g_host[o:o + s.numel] for o, s in zip(M.off, self.specs)]
            self.opt.step_host(views, self.amax_host)
            torch.cuda.synchronize()
            M.g.copy_(self.g_host)  # what the oracle reads
        else:
            self.opt.step()
        if with_oracle:
            self.oracle_step()

    def oracle_step(self) -> None:
        M, t, hp = self.model, self.t, self.hp
        grads = {i: bf16_host_bits(M.view(M.g, i)) for i in self.subset}

        def one(i):
            self.ref[i].step(grads[i], hp["lr"], hp["beta1"], hp["beta2"], hp["eps"],
                             hp["weight_decay"], t, self.flags)

        # ctypes releases the GIL: the oracle runs one tensor per thread
        order = sorted(self.subset, key=lambda i: -self.specs[i].numel)
        with ThreadPoolExecutor(THREADS) as ex:
            list(ex.map(one, order))

    # ---------------------------------------------------------- compare
    def compare(self, max_flip_fraction: float = 0.0) -> dict:
        """Element-wise comparison of the oracle subset, bit for bit: codes,
        params, scales and amax.  With max_flip_fraction > 0 a code may differ
        by one step on at most that fraction of the elements, and the param
        of such an element within 1e-6 relative; by default nothing may
        differ."""
        torch.cuda.synchronize()
        M = self.model
        sm, sv = M.scale_m.cpu().numpy(), M.scale_v.cpu().numpy()
        am, av = M.amax_m.cpu().numpy(), M.amax_v.cpu().numpy()
        total, flips, worst = 0, 0, 0.0
        for i in self.subset:
            r = self.ref[i]
            n = self.specs[i].numel
            total += n
            p = M.view(M.p, i).cpu().numpy()
            m = M.view(M.m, i).cpu().numpy()
            v = M.view(M.v, i).cpu().numpy()
            bad = np.zeros(n, bool)
            for got, exp, fmt in ((m, r.m, self.m_fmt), (v, r.v, self.v_fmt)):
                if fmt == oracle.FP32:
                    eq = (got.view(np.uint32) == exp.view(np.uint32)) | (np.isnan(got) & np.isnan(exp))
                    assert eq.all(), "tensor %d: fp32 moment differs at %s" % (i, np.flatnonzero(~eq)[:8])
                    continue
                # byte for byte: a NaN moment encodes to 0x7F on both sides
                d = np.flatnonzero(got != exp)
                if d.size:
                    assert (np.abs(got[d].astype(np.int32) - exp[d].astype(np.int32)) == 1).all(), \
                        "tensor %d: codes differ by more than one step at %s" % (i, d[:8])
                    bad[d] = True
            flips += int(bad.sum())
            ok = ~bad
            both_nan = np.isnan(p) & np.isnan(r.p)
            close = np.abs(p.astype(np.float64) - r.p) <= 1e-6 * np.abs(r.p.astype(np.float64))
            exact = p.view(np.uint32) == r.p.view(np.uint32)
            okp = exact | both_nan | (bad & close)
            assert okp.all(), "tensor %d: params differ at %s (gpu %s, oracle %s)" % (
                i, np.flatnonzero(~okp)[:8], p[~okp][:4], r.p[~okp][:4])
            if ok.any():
                rel = np.abs(p[ok].astype(np.float64) - r.p[ok]) / np.maximum(np.abs(r.p[ok]), 1e-30)
                rel = rel[np.isfinite(rel)]
                if rel.size:
                    worst = max(worst, float(rel.max()))
            for got, exp, what in ((sm[i], r.scale_m[0], "scale_m"), (sv[i], r.scale_v[0], "scale_v"),
                                   (am[i], r.amax_m[0], "amax_m"), (av[i], r.amax_v[0], "amax_v")):
                assert (np.isnan(got) and np.isnan(exp)) or np.float32(got).view(np.uint32) == \
                    np.float32(exp).view(np.uint32), "tensor %d: %s %r vs oracle %r" % (i, what, got, exp)
        assert flips <= max_flip_fraction * total, "%d code flips in %d elements" % (flips, total)
        return {"elements": total, "flips": flips, "max_rel_param_err": worst}

    def check_invariants(self) -> None:
        """Properties of every tensor (also those the oracle does not run):
        scales are powers of two, amax*scale_next within (max/2, max], params
        finite."""
        torch.cuda.synchronize()
        M = self.model
        for fmt, s, a in ((self.m_fmt, M.scale_m, M.amax_m), (self.v_fmt, M.scale_v, M.amax_v)):
            if fmt == oracle.FP32:
                continue
            s, a = s.cpu().numpy().astype(np.float64), a.cpu().numpy().astype(np.float64)
            assert (np.frexp(s)[0] == 0.5).all(), "scale not a power of two"
            nxt = np.array([pins.pow2scale_bruteforce(fmt, float(x), float(y)) for x, y in zip(a, s)])
            live = (a > 0) & np.isfinite(a) & (np.log2(nxt) > -126) & (np.log2(nxt) < 126)
            prod = a[live] * nxt[live]
            assert ((prod > pins.FMAX[fmt] / 2) & (prod <= pins.FMAX[fmt])).all()
        assert torch.isfinite(M.p).all()

