"""ZeRO-1 step on the GPU against the oracle: the sharded wrapper drives the
CUDA kernels on the rank-blocked buffers, in an NCCL process group of one
rank, and in a gloo group of two ranks sharing the one GPU."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from fp8_quantized_adam_b200 import capi, workloads, zero
from gpu_harness import HP, bf16_host_bits

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_zero1_single_rank_nccl_matches_oracle():
    import torch.distributed as dist

    dev = torch.device("cuda:0")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()), RANK="0", WORLD_SIZE="1")
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev)
    try:
        specs = workloads.custom_layout([70001, 4096, 33, 0, 200003])
        L = zero.ShardLayout([s.numel for s in specs], 1)
        params = torch.zeros(L.total, device=dev)
        workloads.init_params_into(specs, L.views(params), 61)
        grads = torch.zeros(L.total, dtype=torch.bfloat16, device=dev)
        ref = [oracle.TensorState(v.cpu().numpy(), oracle.E4M3, oracle.E5M2) for v in L.views(params)]
        opt = zero.ZeroFP8AdamW(L, params, grads, lr=HP["lr"], betas=(HP["beta1"], HP["beta2"]), eps=HP["eps"],
                                weight_decay=HP["weight_decay"])
        sig = workloads.tensor_sigmas(specs, 61)
        for t in range(1, 4):
            workloads.grads_into(specs, L.views(grads), 61, t, sig)
            opt.step()
            for st, g in zip(ref, L.views(grads)):
                st.step(bf16_host_bits(g), HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t)
        torch.cuda.synchronize()
        for v, st in zip(L.views(params), ref):
            assert (v.cpu().numpy().view(np.uint32) == st.p.view(np.uint32)).all()
        opt.close()
    finally:
        dist.destroy_process_group()


SIZES2 = [70001, 4096, 33, 200003, 5000, 1, 0, 131072 * 2 + 77]


SR2 = {"rn": {}, "sr16": dict(stochastic_rounding=True, sr_draw_bits=16, seed=0xBEEF)}


def _sr_flags(kw):
    if not kw.get("stochastic_rounding"):
        return 0
    return oracle.FLAG_STOCHASTIC | (oracle.FLAG_SR_DRAW16 if kw.get("sr_draw_bits") == 16 else 0)


def _two_rank_worker(rank, world, port, q, sr):
    """One rank: the real CUDA step on its shard (cuda:0, shared with the
    other rank), collectives on host copies over gloo."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK="0")
    try:
        import torch.distributed as dist

        from fp8_quantized_adam_b200 import ranks

        torch.cuda.set_device(0)
        dev = torch.device("cuda:0")
        ranks.init("gloo", timeout_s=120)
        specs = workloads.custom_layout(SIZES2)
        L = zero.ShardLayout([s.numel for s in specs], world)
        params = torch.zeros(L.total, device=dev)
        workloads.init_params_into(specs, L.views(params), 71)  # identical on every rank
        p0 = params.cpu()
        grads = torch.zeros(L.total, dtype=torch.bfloat16, device=dev)
        opt = zero.ZeroFP8AdamW(L, params, grads, collectives=zero.HostCollectives(), lr=HP["lr"],
                                betas=(HP["beta1"], HP["beta2"]), eps=HP["eps"], weight_decay=HP["weight_decay"],
                                **sr)
        sig = workloads.tensor_sigmas(specs, 71)
        reduced = []
        launches0 = capi.fp8adam_launch_count()
        for t in range(1, 4):
            workloads.grads_into(specs, L.views(grads), 71 + 100 * rank, t, sig)  # each rank its own grads
            opt.step()
            torch.cuda.synchronize()
            full = torch.zeros(L.total, dtype=torch.bfloat16)
            dist.all_gather_into_tensor(full, opt.g_block.cpu())
            reduced.append(full)
        launches = capi.fp8adam_launch_count() - launches0
        opt.local.check()
        # the single-process oracle: every tensor, the summed gradients, the 1/world average
        c = oracle.grad_multiplier(0.0, float(world), 0.0)
        ref = [oracle.TensorState(v.numpy(), oracle.E4M3, oracle.E5M2) for v in L.views(p0)]
        for t, full in enumerate(reduced, start=1):
            for i, (st, g) in enumerate(zip(ref, L.views(full))):
                st.step_ex(bf16_host_bits(g), HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t,
                           _sr_flags(sr), grad_mult=c, seed=sr.get("seed", 0), tensor_index=i)
        ph = params.cpu()
        ok = all((v.numpy().view(np.uint32) == st.p.view(np.uint32)).all() for v, st in zip(L.views(ph), ref))
        # this rank's moments, scales and amax
        mine = L.parts[rank]
        loc = opt.local
        for k, i in enumerate(mine):
            st = ref[i]
            ok = ok and (loc.m[k].cpu().numpy() == st.m).all() and (loc.v[k].cpu().numpy() == st.v).all()
            for nm in ("scale_m", "scale_v", "amax_m", "amax_v"):
                ok = ok and np.float32(float(getattr(loc, nm)[k])).view(np.uint32) == getattr(st, nm).view(np.uint32)[0]
        opt.close()
        q.put((rank, bool(ok), len(mine), launches))
        ranks.finish()
    except Exception as ex:  # reported to the parent, which fails the test
        q.put((rank, False, repr(ex), -1))


@pytest.mark.parametrize("sr", list(SR2))
def test_zero1_two_gloo_ranks_run_the_cuda_step(sr):
    """ZeRO-1 at world size 2 with the CUDA step inside it: two processes
    share cuda:0, each runs FP8AdamW on the tensors it owns between a real
    reduce-scatter and all-gather (gloo, on host copies; the ranks' kernels
    never wait on each other).  After three steps every param on every rank,
    and each rank's moment codes, scales and amax, equal a single-process
    oracle run over all tensors on the summed gradients, bit for bit.  The
    1/world average is a constant multiplier: one step kernel per step after
    step 1, no gradient pre-pass.  With stochastic rounding (16-bit draws)
    each shard keys its draws by the tensors' indices in the whole model, so
    the sharded run still equals the single-process one."""
    import torch.multiprocessing as mp

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_two_rank_worker, args=(r, world, port, q, SR2[sr])) for r in range(world)]
    for p in ps:
        p.start()
    res = [q.get(timeout=600) for _ in range(world)]
    for p in ps:
        p.join(timeout=120)
    for rank, ok, owned, launches in res:
        assert ok, (rank, owned)
        assert isinstance(owned, int) and owned >= 1
        # step 1: amax pre-pass + step kernel; steps 2 and 3: the step kernel only
        assert launches == 4, (rank, launches)
