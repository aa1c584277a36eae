"""FP8AdamW: a torch-facing handle on the C-ABI optimizer.

torch owns the device memory (params, grads, moment codes, scales, amax) and
the stream; the step itself is one call into ``libfp8adam.so``.  The state
(params, m/v codes, scales, amax, step count) lives in caller-visible
tensors, so ``state_dict`` / ``load_state_dict`` checkpoint and resume it
bit for bit.
"""
from __future__ import annotations

import ctypes
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

    Options (fp8adam_create_ex): ``margin_m``/``margin_v`` (scale margin),
    ``amax_history_len`` (scale from the max of the last N amax; the ring is
    allocated here and checkpointed), ``update_from_stored`` (the update reads
    the requantised moments), ``stochastic_rounding`` with ``seed`` and
    ``sr_draw_bits`` (32: the integer encoder with 32-bit draws; 16: 16-bit
    draws rounded by the hardware's stochastic-rounding conversion) and
    ``sr_tensor_ids`` (each tensor's word in the random counter, by default
    its position in ``params``; a shard of a larger model passes the
    tensors' indices in the whole model), and
    ``param_bf16`` (bf16 tensors receiving the updated params).  Per step:
    ``step(loss_scale=, max_norm=, skip_nonfinite=)`` (fp8adam_step_ex).
    """

    def __init__(self, params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor], *,
                 lr: float = 3e-4, betas=(0.9, 0.95), eps: float = 1e-8, weight_decay: float = 0.1,
                 m_fmt="e4m3", v_fmt="e5m2", m: Optional[List[torch.Tensor]] = None,
                 v: Optional[List[torch.Tensor]] = None, scale_m: Optional[torch.Tensor] = None,
                 scale_v: Optional[torch.Tensor] = None, amax_m: Optional[torch.Tensor] = None,
                 amax_v: Optional[torch.Tensor] = None, stats: bool = False,
                 jit_every_step: bool = False, margin_m: int = 0, margin_v: int = 0,
                 amax_history_len: int = 0, update_from_stored: bool = False,
                 stochastic_rounding: bool = False, seed: int = 0, sr_draw_bits: int = 32,
                 sr_tensor_ids: Optional[Sequence[int]] = None,
                 param_bf16: Optional[List[torch.Tensor]] = None, chunk_elems: int = 0,
                 tma: bool = True):
        if len(params) == 0 or len(params) != len(grads):
            raise ValueError("need matching, non-empty param and grad lists")
        if sr_draw_bits not in (16, 32):
            raise ValueError("sr_draw_bits is 32 or 16")
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

        def check(bufs, dtype, what):
            # the library reads and writes these through raw pointers: size,
            # dtype, device and layout must be exactly as declared
            if len(bufs) != T:
                raise ValueError("%s: one buffer per param expected" % what)
            for b, p in zip(bufs, self.params):
                if b.dtype != dtype or b.numel() != p.numel() or b.device != dev or not b.is_contiguous():
                    raise ValueError("%s: contiguous %s of %d elements on %s expected" % (what, dtype, p.numel(), dev))

        check(self.m, torch.float32 if self.m_fmt == capi.FP32 else torch.uint8, "m")
        check(self.v, torch.float32 if self.v_fmt == capi.FP32 else torch.uint8, "v")

        def per_tensor(t, fill, what):
            if t is None:
                return torch.full((T,), fill, dtype=torch.float32, device=dev)
            if t.dtype != torch.float32 or t.numel() != T or t.device != dev or not t.is_contiguous():
                raise ValueError("%s: contiguous float32 [%d] on %s expected" % (what, T, dev))
            return t

        self.scale_m = per_tensor(scale_m, 1.0, "scale_m")
        self.scale_v = per_tensor(scale_v, 1.0, "scale_v")
        self.amax_m = per_tensor(amax_m, 0.0, "amax_m")
        self.amax_v = per_tensor(amax_v, 0.0, "amax_v")
        self.lr, self.betas, self.eps, self.weight_decay = lr, tuple(betas), eps, weight_decay
        self.t = 0
        arr = (capi.fp8adam_tensor * T)()
        for i, (p, g, mm, vv) in enumerate(zip(self.params, self.grads, self.m, self.v)):
            arr[i] = capi.fp8adam_tensor(p.data_ptr(), g.data_ptr(), mm.data_ptr(), vv.data_ptr(), p.numel())
        flags = ((capi.FLAG_STATS if stats else 0) | (capi.FLAG_JIT_EVERY_STEP if jit_every_step else 0)
                 | (capi.FLAG_UPDATE_FROM_STORED if update_from_stored else 0)
                 | (capi.FLAG_STOCHASTIC_ROUNDING if stochastic_rounding else 0)
                 | (capi.FLAG_SR_DRAW16 if sr_draw_bits == 16 else 0)
                 | (0 if tma else capi.FLAG_NO_TMA))
        self.amax_history_len = int(amax_history_len)
        self.hist_m = self.hist_v = None
        if self.amax_history_len > 1:
            self.hist_m = torch.zeros(self.amax_history_len, T, dtype=torch.float32, device=dev)
            self.hist_v = torch.zeros(self.amax_history_len, T, dtype=torch.float32, device=dev)
        self.param_bf16 = list(param_bf16) if param_bf16 is not None else None
        bf16_arr = None
        if self.param_bf16 is not None:
            check(self.param_bf16, torch.bfloat16, "param_bf16")
            bf16_arr = (ctypes.c_void_p * T)(*[b.data_ptr() for b in self.param_bf16])
        # the stochastic-rounding stream: part of the checkpointed state's identity
        self.sr_config = {"stochastic_rounding": bool(stochastic_rounding), "seed": int(seed),
                          "sr_draw_bits": int(sr_draw_bits),
                          "sr_tensor_ids": None if sr_tensor_ids is None else [int(i) for i in sr_tensor_ids]}
        ids_arr = None
        if sr_tensor_ids is not None:
            if len(sr_tensor_ids) != T or any(not 0 <= int(i) < (1 << 32) for i in sr_tensor_ids):
                raise ValueError("sr_tensor_ids: one 32-bit unsigned id per tensor")
            ids_arr = (ctypes.c_uint32 * T)(*[int(i) for i in sr_tensor_ids])
        opts = capi.fp8adam_options(self.scale_m.data_ptr(), self.scale_v.data_ptr(), self.amax_m.data_ptr(),
                                    self.amax_v.data_ptr(), self.m_fmt, self.v_fmt, flags, margin_m, margin_v,
                                    self.amax_history_len,
                                    self.hist_m.data_ptr() if self.hist_m is not None else None,
                                    self.hist_v.data_ptr() if self.hist_v is not None else None,
                                    seed, ctypes.cast(bf16_arr, ctypes.c_void_p) if bf16_arr is not None else None,
                                    chunk_elems, ctypes.cast(ids_arr, ctypes.c_void_p) if ids_arr is not None else None)
        with torch.cuda.device(dev):
            self.ctx = capi.fp8adam_create_ex(arr, T, opts)
        self.device = dev

    def _call(self, fn, *args):
        """A C ABI call on the optimizer's device (the library requires the
        device current at create to be current at every call)."""
        with torch.cuda.device(self.device):
            return fn(*args)

    def step(self, stream: Optional[torch.cuda.Stream] = None, lr: Optional[float] = None,
             loss_scale: float = 1.0, max_norm: float = 0.0, skip_nonfinite: bool = False) -> None:
        """One AdamW step on every tensor, queued on ``stream`` (default: the
        current torch stream).  Never synchronises.  ``loss_scale`` divides
        the gradients, ``max_norm`` > 0 clips their global L2 norm,
        ``skip_nonfinite`` skips the whole step on an inf/NaN gradient."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        self.t += 1
        lr = self.lr if lr is None else lr
        if loss_scale == 1.0 and max_norm <= 0.0 and not skip_nonfinite:
            self._call(capi.fp8adam_step, self.ctx, lr, self.betas[0], self.betas[1], self.eps, self.weight_decay, self.t,
                              s.cuda_stream)
        else:
            sp = capi.fp8adam_step_params(lr, self.betas[0], self.betas[1], self.eps, self.weight_decay, self.t,
                                          loss_scale, max_norm, 1 if skip_nonfinite else 0)
            self._call(capi.fp8adam_step_ex, self.ctx, sp, s.cuda_stream)

    def step_host(self, host_grads: Sequence[torch.Tensor], amax_out: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None, lr: Optional[float] = None,
                  loss_scale: float = 1.0, max_norm: float = 0.0, skip_nonfinite: bool = False) -> None:
        """One step whose gradients come from host memory: ``host_grads[i]``
        (a CPU bf16 tensor of tensor i's size, pinned for overlap) is copied
        into tensor i's gradient buffer on the library's copy stream, and the
        step of each group of tensors starts as soon as that group's copies are
        done.  ``amax_out`` (CPU float32 [2 * T], pinned) receives amax_m then
        amax_v.  Asynchronous: keep the host tensors alive and read
        ``amax_out`` only after ``stream`` has been synchronised."""
        if len(host_grads) != len(self.params):
            raise ValueError("one host gradient per tensor")
        ptrs = (ctypes.c_void_p * len(host_grads))()
        for i, (h, p) in enumerate(zip(host_grads, self.params)):
            if h.device.type != "cpu" or h.dtype != torch.bfloat16 or h.numel() != p.numel() or \
                    not h.is_contiguous():
                raise ValueError("host gradient %d: contiguous CPU bf16 of %d elements expected" % (i, p.numel()))
            ptrs[i] = h.data_ptr() if h.numel() else None
        out = 0
        if amax_out is not None:
            if amax_out.device.type != "cpu" or amax_out.dtype != torch.float32 or \
                    amax_out.numel() != 2 * len(self.params) or not amax_out.is_contiguous():
                raise ValueError("amax_out: contiguous CPU float32 of 2 * T elements expected")
            out = amax_out.data_ptr()
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        self.t += 1
        lr = self.lr if lr is None else lr
        sp = capi.fp8adam_step_params(lr, self.betas[0], self.betas[1], self.eps, self.weight_decay, self.t,
                                      loss_scale, max_norm, 1 if skip_nonfinite else 0)
        try:
            self._call(capi.fp8adam_step_host, self.ctx, sp, ptrs, out, s.cuda_stream)
        except capi.Fp8AdamError:
            self.t -= 1
            raise

    def set_schedule(self, lrs: Sequence[float], first_step: Optional[int] = None, loss_scale: float = 1.0,
                     max_norm: float = 0.0, skip_nonfinite: bool = False,
                     stream: Optional[torch.cuda.Stream] = None) -> None:
        """Upload the parameters of steps first_step .. first_step + len(lrs)
        - 1 (default: the step after the last one run) with learning rate
        lrs[k] for step first_step + k, for ``step_scheduled``."""
        first = self.t + 1 if first_step is None else int(first_step)
        steps = [capi.fp8adam_step_params(float(lr), self.betas[0], self.betas[1], self.eps, self.weight_decay,
                                          first + k, loss_scale, max_norm, 1 if skip_nonfinite else 0)
                 for k, lr in enumerate(lrs)]
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        self._call(capi.fp8adam_set_schedule, self.ctx, steps, s.cuda_stream)

    def step_scheduled(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        """The next step of the schedule, with no per-step host state: can be
        captured in a CUDA graph (torch.cuda.graph) and replayed.  ``self.t``
        does not follow graph replays; ``scheduled_step()`` reads the device
        counter."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        self._call(capi.fp8adam_step_scheduled, self.ctx, s.cuda_stream)
        self.t += 1

    def scheduled_step(self, stream: Optional[torch.cuda.Stream] = None) -> int:
        """The step the next scheduled step will run (synchronises the stream)."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        return self._call(capi.fp8adam_get_schedule_step, self.ctx, s.cuda_stream)

    def grad_info(self, stream: Optional[torch.cuda.Stream] = None):
        """(global grad L2 norm, skipped) of the last step with a gradient
        pre-pass (synchronises the stream)."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        return self._call(capi.fp8adam_get_grad_info, self.ctx, s.cuda_stream)

    def check(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        """Raise if a kernel's bounded wait ran out (synchronises the stream)."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        self._call(capi.fp8adam_check, self.ctx, s.cuda_stream)

    def stats(self, stream: Optional[torch.cuda.Stream] = None):
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        return self._call(capi.fp8adam_get_stats, self.ctx, s.cuda_stream)

    def reset_stats(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        self._call(capi.fp8adam_reset_stats, self.ctx, s.cuda_stream)

    # ---- checkpoint / resume ------------------------------------------
    def state_dict(self) -> dict:
        return {"t": self.t, "params": [p.detach().clone() for p in self.params],
                "m": [x.clone() for x in self.m], "v": [x.clone() for x in self.v],
                "scale_m": self.scale_m.clone(), "scale_v": self.scale_v.clone(),
                "amax_m": self.amax_m.clone(), "amax_v": self.amax_v.clone(),
                "m_fmt": self.m_fmt, "v_fmt": self.v_fmt,
                "amax_history_m": None if self.hist_m is None else self.hist_m.clone(),
                "amax_history_v": None if self.hist_v is None else self.hist_v.clone(),
                "sr_config": dict(self.sr_config)}

    def load_state_dict(self, sd: dict) -> None:
        if sd["m_fmt"] != self.m_fmt or sd["v_fmt"] != self.v_fmt:
            raise ValueError("moment formats differ")
        if "sr_config" in sd and sd["sr_config"] != self.sr_config:
            # the draws of step t depend on the seed, the draw width and the
            # tensor ids: a different stream would not continue the run
            raise ValueError("stochastic-rounding configuration differs: %r vs %r" % (sd["sr_config"],
                                                                                       self.sr_config))
        with torch.no_grad():
            for dst, src in zip(self.params, sd["params"]):
                dst.copy_(src)
            for dst, src in zip(self.m, sd["m"]):
                dst.copy_(src)
            for dst, src in zip(self.v, sd["v"]):
                dst.copy_(src)
            for name in ("scale_m", "scale_v", "amax_m", "amax_v"):
                getattr(self, name).copy_(sd[name])
            if self.hist_m is not None:
                self.hist_m.copy_(sd["amax_history_m"])
                self.hist_v.copy_(sd["amax_history_v"])
        self.t = int(sd["t"])

    def close(self) -> None:
        if getattr(self, "ctx", None):
            self._call(capi.fp8adam_destroy, self.ctx)
            self.ctx = None

    def __del__(self):  # pragma: no cover - best effort
        try:
            self.close()
        except Exception:
            pass
