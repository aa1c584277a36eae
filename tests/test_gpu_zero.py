"""ZeRO-1 step on the GPU (NCCL process group of one rank) against the oracle:
the sharded wrapper drives the CUDA kernels on the rank-blocked buffers."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from fp8_quantized_adam_b200 import workloads, zero
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
