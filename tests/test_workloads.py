"""The seeded synthetic inputs (fp8_quantized_adam_b200/workloads.py) against
the configurations they stand in for: layout sizes and shapes, offsets, and
the value distributions of params and gradients (CPU)."""
import math

import numpy as np
import torch

from fp8_quantized_adam_b200 import workloads


def test_layout_sizes_match_the_configurations():
    cases = {"single_1m": (1, 1_048_576), "llama2_100m": (110, 109_529_856),
             "llama2_7b": (291, 6_738_415_616), "stress_20k": (20_008, 2_229_403_648)}
    for name, (tensors, params) in cases.items():
        specs = workloads.layout(name)
        assert len(specs) == tensors and workloads.total_params(specs) == params, name


def test_llama_layouts_have_the_model_shapes():
    # Llama2-100M: d 768, 12 layers, SwiGLU FFN 2048, vocab 32000, tied embedding
    s = {t.name: t for t in workloads.layout("llama2_100m")}
    assert s["embed"].numel == 32000 * 768 and "lm_head" not in s
    assert s["l0.q"].numel == 768 * 768 and s["l11.w1"].numel == 768 * 2048 and s["l11.w2"].numel == 2048 * 768
    assert s["l5.attn_norm"].numel == 768 and s["final_norm"].kind == "norm"
    # Llama2-7B: d 4096, 32 layers, FFN 11008, untied embedding / LM head
    s = {t.name: t for t in workloads.layout("llama2_7b")}
    assert s["embed"].numel == s["lm_head"].numel == 32000 * 4096
    assert s["l31.w3"].numel == 4096 * 11008 and "l32.q" not in s


def test_offsets_are_aligned_and_disjoint():
    specs = workloads.custom_layout([0, 1, 63, 64, 65, 4097])
    off = workloads.offsets(specs)
    assert all(o % workloads.ALIGN_ELEMS == 0 for o in off)
    for i, s in enumerate(specs):
        assert off[i] + s.numel <= off[i + 1]


def _grads(specs, cfg, step, sig=None):
    views = [torch.empty(s.numel, dtype=torch.bfloat16) for s in specs]
    workloads.grads_into(specs, views, cfg, step, sig)
    return [v.float().numpy().astype(np.float64) for v in views]


def test_draws_are_seeded_and_change_per_step():
    specs = workloads.custom_layout([5000, 300])
    a, b, c = _grads(specs, 9, 1), _grads(specs, 9, 1), _grads(specs, 9, 2)
    assert all((x == y).all() for x, y in zip(a, b))
    assert not (a[0] == c[0]).all()
    pa = [torch.empty(s.numel) for s in specs]
    pb = [torch.empty(s.numel) for s in specs]
    workloads.init_params_into(specs, pa, 9)
    workloads.init_params_into(specs, pb, 9)
    assert all(torch.equal(x, y) for x, y in zip(pa, pb))


def test_param_and_gradient_distributions():
    # params N(0, 0.02); norm gains 1.0
    specs = [workloads.TensorSpec("w", 400_000, "matrix"), workloads.TensorSpec("n", 768, "norm")]
    views = [torch.empty(s.numel) for s in specs]
    workloads.init_params_into(specs, views, 3)
    assert abs(float(views[0].std()) / 0.02 - 1.0) < 0.01 and abs(float(views[0].mean())) < 1e-3
    assert (views[1] == 1.0).all()
    # heavy-tailed matrix grads: N(0, sigma_t), sigma_t = 10^U(-5,-2), 0.1% of elements x100
    sig = workloads.tensor_sigmas(workloads.layout("llama2_100m"), 2)
    assert all(1e-5 <= x <= 1e-2 for x in sig) and len(set(sig)) == len(sig)
    g = _grads(specs[:1], 2, 1, [1e-3])[0]
    outliers = np.abs(g) > 1e-3 * 8  # beyond 8 sigma: only the x100 draws
    assert 0.0005 < outliers.mean() < 0.0015
    assert abs(np.std(g[~outliers]) / 1e-3 - 1.0) < 0.02
    # the single-tensor config: g = 10^U(-6,-1) * N(0,1), per element (spans 5 decades)
    g = _grads([workloads.TensorSpec("w", 200_000, "single")], 1, 1)[0]
    lg = np.log10(np.abs(g[g != 0]))
    assert lg.max() < 0.5 and np.quantile(lg, 0.5) < -3.0 and np.quantile(lg, 0.99) > -1.5
    # the stress config's small tensors: N(0, 1e-4)
    g = _grads([workloads.TensorSpec("s", 200_000, "small")], 5, 1)[0]
    assert abs(np.std(g) / 1e-4 - 1.0) < 0.02 and math.isclose(np.mean(g), 0.0, abs_tol=2e-6)
