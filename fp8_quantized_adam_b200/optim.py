"""FP8AdamW: a torch-facing handle on the C-ABI optimizer.

torch owns the device memory (params, grads, moment codes, scales, amax) and
the stream; the step itself is one call into ``libfp8adam.so``.  The state
(params, m/v codes, scales, amax, step count) lives in caller-visible
tensors, so ``state_dict`` / ``load_state_dict`` checkpoint and resume it
bit for bit.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from . import capi

FMT_IDS = {"e4m3": capi.E4M3, "e5m2": capi.E5M2, "fp32": capi.FP32}


def _fmt_id(f) -> int:
    return FMT_IDS[f] if isinstance(f, str) else int(f)


class FP8AdamW:
    """AdamW with FP8-stored moments over a list of CUDA tensors.

    params: fp32 tensors; grads: bf16 tensors of the same sizes.  m/v are
    allocated (zeros) unless given; ``m_fmt``/``v_fmt`` default to E4M3/E5M2.
    The tensors must keep their storage (addresses) for the optimizer's
    lifetime.
    """

    def __init__(self, params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor], *,
                 lr: float = 3e-4, betas=(0.9, 0.95), eps: float = 1e-8, weight_decay: float = 0.1,
                 m_fmt="e4m3", v_fmt="e5m2", m: Optional[List[torch.Tensor]] = None,
                 v: Optional[List[torch.Tensor]] = None, scale_m: Optional[torch.Tensor] = None,
                 scale_v: Optional[torch.Tensor] = None, amax_m: Optional[torch.Tensor] = None,
                 amax_v: Optional[torch.Tensor] = None, stats: bool = False,
                 jit_every_step: bool = False):
        if len(params) == 0 or len(params) != len(grads):
            raise ValueError("need matching, non-empty param and grad lists")
        self.params, self.grads = list(params), list(grads)
        dev = self.params[0].device
        if dev.type != "cuda":
            raise ValueError("FP8AdamW runs on CUDA tensors only")
        self.m_fmt, self.v_fmt = _fmt_id(m_fmt), _fmt_id(v_fmt)
        for p, g in zip(self.params, self.grads):
            if p.dtype != torch.float32 or g.dtype != torch.bfloat16 or p.numel() != g.numel():
                raise ValueError("params must be fp32 and grads bf16 of the same size")
            if not (p.is_contiguous() and g.is_contiguous()) or p.device != dev or g.device != dev:
                raise ValueError("params and grads must be contiguous tensors on one device")

        def moments(given, fmt):
            if given is not None:
                return list(given)
            dt = torch.float32 if fmt == capi.FP32 else torch.uint8
            return [torch.zeros(p.numel(), dtype=dt, device=dev) for p in self.params]

        self.m = moments(m, self.m_fmt)
        self.v = moments(v, self.v_fmt)
        T = len(self.params)
        self.scale_m = scale_m if scale_m is not None else torch.ones(T, dtype=torch.float32, device=dev)
        self.scale_v = scale_v if scale_v is not None else torch.ones(T, dtype=torch.float32, device=dev)
        self.amax_m = amax_m if amax_m is not None else torch.zeros(T, dtype=torch.float32, device=dev)
        self.amax_v = amax_v if amax_v is not None else torch.zeros(T, dtype=torch.float32, device=dev)
        self.lr, self.betas, self.eps, self.weight_decay = lr, tuple(betas), eps, weight_decay
        self.t = 0
        arr = (capi.fp8adam_tensor * T)()
        for i, (p, g, mm, vv) in enumerate(zip(self.params, self.grads, self.m, self.v)):
            arr[i] = capi.fp8adam_tensor(p.data_ptr(), g.data_ptr(), mm.data_ptr(), vv.data_ptr(), p.numel())
        flags = (capi.FLAG_STATS if stats else 0) | (capi.FLAG_JIT_EVERY_STEP if jit_every_step else 0)
        with torch.cuda.device(dev):
            self.ctx = capi.fp8adam_create(arr, T, self.scale_m.data_ptr(), self.scale_v.data_ptr(),
                                           self.amax_m.data_ptr(), self.amax_v.data_ptr(),
                                           self.m_fmt, self.v_fmt, flags)
        self.device = dev

    def step(self, stream: Optional[torch.cuda.Stream] = None, lr: Optional[float] = None) -> None:
        """One AdamW step on every tensor, queued on ``stream`` (default: the
        current torch stream).  Never synchronises."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        self.t += 1
        capi.fp8adam_step(self.ctx, self.lr if lr is None else lr, self.betas[0], self.betas[1], self.eps,
                          self.weight_decay, self.t, s.cuda_stream)

    def stats(self, stream: Optional[torch.cuda.Stream] = None):
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        return capi.fp8adam_get_stats(self.ctx, s.cuda_stream)

    def reset_stats(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        capi.fp8adam_reset_stats(self.ctx, s.cuda_stream)

    # ---- checkpoint / resume ------------------------------------------
    def state_dict(self) -> dict:
        return {"t": self.t, "params": [p.detach().clone() for p in self.params],
                "m": [x.clone() for x in self.m], "v": [x.clone() for x in self.v],
                "scale_m": self.scale_m.clone(), "scale_v": self.scale_v.clone(),
                "amax_m": self.amax_m.clone(), "amax_v": self.amax_v.clone(),
                "m_fmt": self.m_fmt, "v_fmt": self.v_fmt}

    def load_state_dict(self, sd: dict) -> None:
        if sd["m_fmt"] != self.m_fmt or sd["v_fmt"] != self.v_fmt:
            raise ValueError("moment formats differ")
        with torch.no_grad():
            for dst, src in zip(self.params, sd["params"]):
                dst.copy_(src)
            for dst, src in zip(self.m, sd["m"]):
                dst.copy_(src)
            for dst, src in zip(self.v, sd["v"]):
                dst.copy_(src)
            for name in ("scale_m", "scale_v", "amax_m", "amax_v"):
                getattr(self, name).copy_(sd[name])
        self.t = int(sd["t"])

    def close(self) -> None:
        if getattr(self, "ctx", None):
            capi.fp8adam_destroy(self.ctx)
            self.ctx = None

    def __del__(self):  # pragma: no cover - best effort
        try:
            self.close()
        except Exception:
            pass
