"""The CUDA step against the oracle, element by element, free-running from
the same seeded state on the same seeded gradients (all calls go through the
C ABI)."""
import math

import numpy as np
import pytest
import torch

import oracle
from fp8_quantized_adam_b200 import FP8AdamW, capi, workloads
from gpu_harness import HP, Run, bf16_host_bits

pytestmark = pytest.mark.gpu

E4, E5, F32 = oracle.E4M3, oracle.E5M2, oracle.FP32


def test_single_tensor_1m_all_elements_10_steps():
    """1,048,576 params, g = 10^U(-6,-1) * N(0,1): every element, 10 steps."""
    r = Run(workloads.layout("single_1m"), workloads.CFG_ID["single_1m"])
    for _ in range(10):
        r.step()
        res = r.compare()
    assert res["flips"] == 0


def test_llama2_100m_layout_subset_100_steps():
    specs = workloads.layout("llama2_100m")
    names = [s.name for s in specs]
    subset = [i for i, s in enumerate(specs) if s.kind == "norm"] + [names.index("l0.q"), names.index("l5.w1")]
    r = Run(specs, workloads.CFG_ID["llama2_100m"], subset=subset)
    for t in range(1, 101):
        r.step()
        if t in (1, 2, 3, 10, 50, 100):
            r.compare()
            r.check_invariants()


@pytest.mark.slow
def test_format_ablation_all_modes_200_steps():
    """The format-ablation configuration over its full 200 steps: the five
    (m, v) storage modes in lockstep on the same seeded gradients of the
    Llama2-100M layout (the Fig. 5 moment-format ablation of the explainer's
    "实验证据" section; its v-in-E4M3 modes run away, which is where a late code
    difference would show).  Per mode the whole layout steps in one context,
    as the ablation report runs it.  A second context per mode holds only the
    oracle's subset (two projection matrices, two norms): tensors are
    independent, so it must match the whole run bit for bit, and its counters
    give the subset's flushed-v and saturated counts, compared with the
    oracle's at every step.  Codes, scales and amax equal the oracle's byte
    for byte every 20 steps, and so are the params.  At the end, Fig. 5's
    outcome: (E4M3, E5M2) drifts least from the fp32-moment run."""
    specs = workloads.layout("ablation_100m")
    cfg = workloads.CFG_ID["ablation_100m"]
    names = [s.name for s in specs]
    subset = [names.index(n) for n in ("l3.k", "l11.w3", "l5.attn_norm", "final_norm")]
    dev = torch.device("cuda:0")
    sig = workloads.tensor_sigmas(specs, cfg)
    g = workloads.FlatModel(specs, dev).g  # one gradient buffer for every mode
    off = workloads.offsets(specs)
    gviews = [g[off[i]:off[i] + s.numel] for i, s in enumerate(specs)]
    modes = [(E4, E4), (E4, E5), (E5, E4), (E5, E5), (F32, F32)]
    runs = []
    for mf, vf in modes:
        M = workloads.FlatModel(specs, dev, m_fp32=mf == F32, v_fp32=vf == F32)
        workloads.init_params_into(specs, M.views(M.p), cfg)
        whole = FP8AdamW(M.views(M.p), gviews, m_fmt=mf, v_fmt=vf, m=M.views(M.m), v=M.views(M.v),
                         scale_m=M.scale_m, scale_v=M.scale_v, amax_m=M.amax_m, amax_v=M.amax_v)
        sub_specs = [specs[i] for i in subset]
        S = workloads.FlatModel(sub_specs, dev, m_fp32=mf == F32, v_fp32=vf == F32)
        for k, i in enumerate(subset):
            S.view(S.p, k).copy_(M.view(M.p, i))
        part = FP8AdamW(S.views(S.p), [gviews[i] for i in subset], m_fmt=mf, v_fmt=vf, m=S.views(S.m),
                        v=S.views(S.v), scale_m=S.scale_m, scale_v=S.scale_v, amax_m=S.amax_m, amax_v=S.amax_v,
                        stats=True)
        torch.cuda.synchronize()
        ref = [oracle.TensorState(M.view(M.p, i).cpu().numpy(), mf, vf) for i in subset]
        runs.append((mf, vf, M, whole, S, part, ref))
    hp = HP
    jobs = [(r, k) for r in range(len(runs)) for k in range(len(subset))]
    jobs.sort(key=lambda rk: -specs[subset[rk[1]]].numel)
    checkpoints = {1, 2} | set(range(20, 201, 20))
    flushed_seen = {}
    from concurrent.futures import ThreadPoolExecutor

    with ThreadPoolExecutor(16) as ex:
        for t in range(1, 201):
            workloads.grads_into(specs, gviews, cfg, t, sig)
            for (_, _, _, whole, _, part, _) in runs:
                whole.step()
                part.reset_stats()
                part.step()
            bits = [bf16_host_bits(gviews[i]) for i in subset]
            before = [[st.stats.copy() for st in run[6]] for run in runs]

            def one(rk):
                r, k = rk
                runs[r][6][k].step(bits[k], hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"], t)

            list(ex.map(one, jobs))
            for r, (mf, vf, M, whole, S, part, ref) in enumerate(runs):
                exp = tuple(int(sum(int(st.stats[c]) - int(b[c]) for st, b in zip(ref, before[r]))) for c in (0, 1))
                assert part.stats() == exp, (t, mf, vf, part.stats(), exp)
                if mf != F32:
                    flushed_seen[(mf, vf)] = flushed_seen.get((mf, vf), 0) + exp[0]
            if t not in checkpoints:
                continue
            torch.cuda.synchronize()
            for mf, vf, M, whole, S, part, ref in runs:
                for k, i in enumerate(subset):
                    for buf_s, buf_m in ((S.p, M.p), (S.m, M.m), (S.v, M.v)):
                        assert torch.equal(S.view(buf_s, k).view(torch.uint8) if buf_s.dtype == torch.uint8 else
                                           S.view(buf_s, k).view(torch.int32),
                                           M.view(buf_m, i).view(torch.uint8) if buf_m.dtype == torch.uint8 else
                                           M.view(buf_m, i).view(torch.int32)), (t, mf, vf, i)
                    st = ref[k]
                    for got, exp_ in ((M.view(M.m, i), st.m), (M.view(M.v, i), st.v)):
                        got = got.cpu().numpy()
                        assert got.view(np.uint8).tobytes() == exp_.view(np.uint8).tobytes(), (t, mf, vf, i)
                    for nm, arr in (("scale_m", M.scale_m), ("scale_v", M.scale_v), ("amax_m", M.amax_m),
                                    ("amax_v", M.amax_v)):
                        assert np.float32(float(arr[i])).view(np.uint32) == getattr(st, nm).view(np.uint32)[0], \
                            (t, mf, vf, i, nm)
                    p = M.view(M.p, i).cpu().numpy()
                    assert (p.view(np.uint32) == st.p.view(np.uint32)).all(), (t, mf, vf, i)
    # Fig. 5's outcome over the whole layout (expected, not a bit-level pin):
    # against the fp32-moment run, the pair the paper chose, m in E4M3 and v
    # in E5M2, drifts least, and both pairs with v in E4M3 drift far more
    # than both with v in E5M2
    torch.cuda.synchronize()
    p32 = runs[-1][2].p
    dp = {(mf, vf): float((M.p - p32).abs().max()) for mf, vf, M, *_ in runs[:-1]}
    assert dp[(E4, E5)] == min(dp.values()), dp
    assert min(dp[(E4, E4)], dp[(E5, E4)]) > 10 * max(dp[(E4, E5)], dp[(E5, E5)]), dp
    for run in runs:
        run[3].close()
        run[5].close()
    # Fig. 5's mechanism: v stored in E4M3 flushes far more than in E5M2
    assert flushed_seen[(E4, E4)] > 10 * flushed_seen[(E4, E5)]


def test_stats_counters_match_oracle():
    """Flushed-v and saturation counters over a whole model equal the sums of
    the oracle's per-tensor counters; v in E4M3 flushes more than E5M2."""
    specs = workloads.custom_layout([70001, 4096, 33, 200000])
    flushed = {}
    for vf in (E4, E5):
        r = Run(specs, 9, m_fmt=E4, v_fmt=vf, stats=True)
        for t in range(1, 6):
            r.step()
        r.compare()
        got = r.opt.stats()
        exp = tuple(int(sum(int(r.ref[i].stats[k]) for i in r.subset)) for k in (0, 1))
        assert got == exp
        flushed[vf] = got[0]
    assert flushed[E4] > flushed[E5]


def test_current_scaling_every_step():
    specs = workloads.custom_layout([65536 * 3 + 5, 1000])
    r = Run(specs, 11, jit_every_step=True)
    for _ in range(6):
        r.step()
        r.compare()


def test_edge_sizes_and_misaligned_views():
    """Sizes around the 16-element vector, the 4096-element tile and the
    chunk lengths the library picks (8192 .. 131072), an empty tensor, and
    tensors whose buffers are offset by one element (element-by-element
    path)."""
    sizes = [0, 1, 15, 16, 17, 4095, 4096, 4097, 16383, 16385, 65535, 65536, 65537, 131071, 131073,
             3 * 65536 + 4099]
    specs = workloads.custom_layout(sizes)
    r = Run(specs, 12)
    for _ in range(4):
        r.step()
        r.compare()
    # misaligned: views starting one element into each buffer
    dev = torch.device("cuda:0")
    ns = [33, 4097, 70000]
    p = [torch.zeros(n + 1, device=dev)[1:] for n in ns]
    g = [torch.zeros(n + 1, device=dev, dtype=torch.bfloat16)[1:] for n in ns]
    m = [torch.zeros(n + 1, device=dev, dtype=torch.uint8)[1:] for n in ns]
    v = [torch.zeros(n + 1, device=dev, dtype=torch.uint8)[1:] for n in ns]
    specs2 = workloads.custom_layout(ns)
    workloads.init_params_into(specs2, p, 13)
    opt = FP8AdamW(p, g, m=m, v=v)
    ref = [oracle.TensorState(x.cpu().numpy(), E4, E5) for x in p]
    sig = workloads.tensor_sigmas(specs2, 13)
    for t in range(1, 4):
        workloads.grads_into(specs2, g, 13, t, sig)
        opt.step()
        for i, rs in enumerate(ref):
            rs.step(bf16_host_bits(g[i]), HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t)
    torch.cuda.synchronize()
    for i, rs in enumerate(ref):
        assert (m[i].cpu().numpy() == rs.m).all() and (v[i].cpu().numpy() == rs.v).all()
        assert (p[i].cpu().numpy().view(np.uint32) == rs.p.view(np.uint32)).all()
        assert float(opt.amax_m[i]) == float(rs.amax_m[0]) and float(opt.scale_v[i]) == float(rs.scale_v[0])


@pytest.mark.parametrize("chunk", [4096, 16384, 131072])
def test_results_do_not_depend_on_the_chunk_length(chunk):
    specs = workloads.custom_layout([300001, 4096, 17, 131072 * 2 + 3])
    runs = []
    for ce in (0, chunk):
        M = workloads.FlatModel(specs, torch.device("cuda:0"))
        workloads.init_params_into(specs, M.views(M.p), 19)
        opt = FP8AdamW(M.views(M.p), M.views(M.g), m=M.views(M.m), v=M.views(M.v), scale_m=M.scale_m,
                       scale_v=M.scale_v, amax_m=M.amax_m, amax_v=M.amax_v, chunk_elems=ce)
        sig = workloads.tensor_sigmas(specs, 19)
        for t in range(1, 5):
            workloads.grads_into(specs, M.views(M.g), 19, t, sig)
            opt.step()
        torch.cuda.synchronize()
        runs.append(M)
    for name in ("p", "m", "v", "scale_m", "scale_v", "amax_m", "amax_v"):
        assert torch.equal(getattr(runs[0], name).view(torch.uint8), getattr(runs[1], name).view(torch.uint8)), name


@pytest.mark.parametrize("fmts", [(E4, E5), (E4, E4), (E5, E4), (E5, E5)], ids=["m4v5", "m4v4", "m5v4", "m5v5"])
def test_tma_staged_and_vector_paths_agree(fmts):
    """The shared-memory (TMA bulk copy) path and the per-thread vector path
    give identical state, counters included, on ragged sizes; the device
    error word stays clear."""
    specs = workloads.custom_layout([300001, 4096, 17, 131072 * 2 + 2049, 2048, 2047, 6144 + 16])
    runs = []
    for tma in (True, False):
        M = workloads.FlatModel(specs, torch.device("cuda:0"))
        workloads.init_params_into(specs, M.views(M.p), 23)
        opt = FP8AdamW(M.views(M.p), M.views(M.g), m_fmt=fmts[0], v_fmt=fmts[1], m=M.views(M.m), v=M.views(M.v),
                       scale_m=M.scale_m, scale_v=M.scale_v, amax_m=M.amax_m, amax_v=M.amax_v, stats=True,
                       tma=tma, chunk_elems=16384)
        sig = workloads.tensor_sigmas(specs, 23)
        for t in range(1, 6):
            workloads.grads_into(specs, M.views(M.g), 23, t, sig)
            opt.step()
        opt.check()
        runs.append((M, opt.stats()))
    for name in ("p", "m", "v", "scale_m", "scale_v", "amax_m", "amax_v"):
        assert torch.equal(getattr(runs[0][0], name).view(torch.uint8), getattr(runs[1][0], name).view(torch.uint8)), name
    assert runs[0][1] == runs[1][1]


def test_back_to_back_steps_match_oracle():
    """Eight steps queued back to back on one stream with nothing in between
    (fixed gradients): with programmatic dependent launch each step's grid
    may start while the previous one finishes, and must still read params,
    moments, scales and amax only after that one's writes.  Every element
    against the oracle after the eighth step, on a layout with long, short
    and one-tile chunks."""
    specs = workloads.custom_layout([3 * 131072 + 77, 4096, 17, 2048 * 9, 70001, 1 << 20])
    r = Run(specs, 29)
    r.draw_grads(1)
    torch.cuda.synchronize()
    for t in range(1, 9):
        r.t = t
        r.opt.step()
    r.opt.check()
    M = r.model
    grads = {i: bf16_host_bits(M.view(M.g, i)) for i in r.subset}
    for t in range(1, 9):
        for i in r.subset:
            r.ref[i].step(grads[i], HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t)
    res = r.compare()
    assert res["flips"] == 0


def test_zero_gradients_keep_scale_and_decay_params():
    specs = workloads.custom_layout([5000])
    r = Run(specs, 14)
    for t in range(1, 4):
        r.t += 1
        r.model.g.zero_()
        r.opt.step()
        r.oracle_step()
        r.compare()
    assert float(r.model.scale_m[0]) == 1.0 and float(r.model.amax_m[0]) == 0.0


def test_nan_gradient_reaches_amax_without_fault():
    specs = workloads.custom_layout([10000, 300])
    r = Run(specs, 15)
    r.step()
    r.t += 1
    r.draw_grads(r.t)
    r.model.g[1234] = float("nan")
    r.opt.step()
    r.oracle_step()
    r.compare()
    assert math.isnan(float(r.model.amax_m[0])) and math.isfinite(float(r.model.amax_m[1]))
    r.step()  # a NaN amax keeps the previous scale; the NaN element stays NaN
    r.compare()


def test_checkpoint_resume_is_bitwise():
    specs = workloads.custom_layout([100000, 4096, 77])
    a = Run(specs, 16, subset=[])
    for _ in range(10):
        a.step(with_oracle=False)
    b = Run(specs, 16, subset=[])
    for _ in range(5):
        b.step(with_oracle=False)
    sd = b.opt.state_dict()
    c = Run(specs, 16, subset=[])  # a fresh optimizer on fresh buffers, then restore
    c.opt.load_state_dict(sd)
    c.t = b.t
    for _ in range(5):
        c.step(with_oracle=False)
    torch.cuda.synchronize()
    for x, y in ((a.model.p, c.model.p), (a.model.m, c.model.m), (a.model.v, c.model.v),
                 (a.model.scale_m, c.model.scale_m), (a.model.amax_v, c.model.amax_v)):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_two_runs_are_bitwise_identical():
    specs = workloads.layout("single_1m")
    runs = []
    for _ in range(2):
        r = Run(specs, 1, subset=[])
        for _ in range(5):
            r.step(with_oracle=False)
        torch.cuda.synchronize()
        runs.append(r)
    for name in ("p", "m", "v", "scale_m", "scale_v", "amax_m", "amax_v"):
        assert torch.equal(getattr(runs[0].model, name).view(torch.uint8),
                           getattr(runs[1].model, name).view(torch.uint8)), name


def test_step_argument_errors_queue_nothing():
    specs = workloads.custom_layout([64])
    r = Run(specs, 17, subset=[])
    before = capi.fp8adam_launch_count()
    for kw in (dict(step=0), dict(beta1=1.0), dict(beta2=-0.1), dict(eps=-1.0), dict(lr=float("nan"))):
        args = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.0, step=1)
        args.update(kw)
        with pytest.raises(capi.Fp8AdamError) as e:
            capi.fp8adam_step(r.opt.ctx, args["lr"], args["beta1"], args["beta2"], args["eps"],
                              args["weight_decay"], args["step"], 0)
        assert e.value.code == capi.ERR_INVALID_ARG
    assert capi.fp8adam_launch_count() == before


@pytest.mark.slow
def test_int64_indexing_beyond_2_pow_31():
    """A 2^31 + 3*4096 + 5 element tensor with inputs periodic in 4096
    elements: outputs are periodic too, so elements past index 2^31 must
    equal the oracle run on one period (same amax, same per-element math)."""
    period = 4096
    n = (1 << 31) + 3 * period + 5
    dev = torch.device("cuda:0")
    base_specs = workloads.custom_layout([period])
    pp = torch.zeros(period)
    workloads.init_params_into(base_specs, [pp], 18)
    sig = workloads.tensor_sigmas(base_specs, 18)
    gg = [torch.zeros(period, dtype=torch.bfloat16) for _ in range(2)]
    for t in (1, 2):
        workloads.grads_into(base_specs, [gg[t - 1]], 18, t, sig)
    reps = (n + period - 1) // period
    p = pp.to(dev).repeat(reps)[:n].contiguous()
    g = torch.empty(n, dtype=torch.bfloat16, device=dev)
    m = torch.zeros(n, dtype=torch.uint8, device=dev)
    v = torch.zeros(n, dtype=torch.uint8, device=dev)
    opt = FP8AdamW([p], [g], m=[m], v=[v])
    ref = oracle.TensorState(pp.numpy(), E4, E5)
    for t in (1, 2):
        g.copy_(gg[t - 1].to(dev).repeat(reps)[:n])
        opt.step()
        ref.step(bf16_host_bits(gg[t - 1]), HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t)
    torch.cuda.synchronize()
    for start in ((1 << 31) - period, (1 << 31), n - 5 - period):
        k = start - start % period
        assert (m[k:k + period].cpu().numpy() == ref.m).all()
        assert (v[k:k + period].cpu().numpy() == ref.v).all()
        assert (p[k:k + period].cpu().numpy().view(np.uint32) == ref.p.view(np.uint32)).all()
    tail = n - (n // period) * period
    assert (m[n - tail:].cpu().numpy() == ref.m[:tail]).all()
    assert float(opt.amax_m[0]) == float(ref.amax_m[0]) and float(opt.scale_v[0]) == float(ref.scale_v[0])


@pytest.mark.slow
def test_stress_20k_tensors_full_parity_2_steps():
    """20,000 x 4096 + 8 x 2^28 in one launch per step; every element of
    every tensor against the oracle (run on all host cores)."""
    r = Run(workloads.layout("stress_20k"), workloads.CFG_ID["stress_20k"])
    for _ in range(2):
        r.step()
        res = r.compare()
    assert res["elements"] == workloads.total_params(r.specs)


def test_stress_20k_tensors_50_steps_subset():
    """The stress configuration's 50 steps (20,000 x 4096 + 8 x 2^28, one
    launch per step); 300 of the small tensors, spread over the list,
    against the oracle at steps 1, 2, 10, 25 and 50 (tensors are independent,
    so a subset check is exact), and the scale invariants of every tensor."""
    specs = workloads.layout("stress_20k")
    small = [i for i, s in enumerate(specs) if s.numel == 4096]
    subset = small[::len(small) // 300][:300]
    r = Run(specs, workloads.CFG_ID["stress_20k"], subset=subset)
    for t in range(1, 51):
        r.step(with_oracle=True)
        if t in (1, 2, 10, 25, 50):
            r.compare()
            r.check_invariants()


@pytest.mark.slow
def test_llama2_7b_layout_subset_bench_length():
    """The 7B-shaped layout over the benchmark's run length (5 warm-up and 20
    timed steps): every tensor steps in one launch per step, and every norm
    gain, l0.q and l31.w2 (62 M params) are compared with the oracle; the
    scale invariants hold for all 291 tensors."""
    specs = workloads.layout("llama2_7b")
    names = [s.name for s in specs]
    subset = [i for i, s in enumerate(specs) if s.kind == "norm"] + [names.index("l0.q"), names.index("l31.w2")]
    r = Run(specs, workloads.CFG_ID["llama2_7b"], subset=subset)
    for t in range(1, 26):
        r.step()
        if t in (1, 2, 3, 5, 10, 15, 20, 25):
            res = r.compare()
            r.check_invariants()
            assert res["flips"] == 0
    r.opt.check()


HOST_LAYOUTS = {"ragged": [70001, 0, 4096, 33, 3 * 65536 + 4099, 17, 200003, 1, 131072, 65535, 9000, 4097],
                "empty_first": [0, 0, 0, 5000, 0, 17, 300000, 0]}


@pytest.mark.parametrize("layout", list(HOST_LAYOUTS))
@pytest.mark.parametrize("jit", [False, True], ids=["delayed", "jit_every_step"])
def test_step_from_host_buffers(jit, layout):
    """fp8adam_step_host: gradients copied from pinned host memory by the
    library (the device buffer is zeroed before each step), the step of each
    tensor group overlapping the copies of the next groups; every element
    against the oracle, and the amax read back to the host.  With empty
    tensors first, the first group that launches clears the JIT amax."""
    sizes = HOST_LAYOUTS[layout]
    specs = workloads.custom_layout(sizes)
    r = Run(specs, 14, host=True, jit_every_step=jit)
    for _ in range(4):
        r.step()
        r.compare()
        M = r.model
        assert torch.equal(r.amax_host[:len(specs)], M.amax_m.cpu()) and \
            torch.equal(r.amax_host[len(specs):], M.amax_v.cpu())


def test_binding_rejects_mismatched_buffers():
    """The torch binding checks every buffer it hands to the library: moment
    dtype and size, per-tensor arrays, bf16 outputs."""
    dev = torch.device("cuda:0")
    p = [torch.zeros(100, device=dev)]
    g = [torch.zeros(100, device=dev, dtype=torch.bfloat16)]
    with pytest.raises(ValueError):
        FP8AdamW(p, g, m=[torch.zeros(100, device=dev)])                        # fp32 m for E4M3
    with pytest.raises(ValueError):
        FP8AdamW(p, g, v=[torch.zeros(99, device=dev, dtype=torch.uint8)])     # wrong size
    with pytest.raises(ValueError):
        FP8AdamW(p, g, scale_m=torch.ones(2, device=dev))                      # T = 1
    with pytest.raises(ValueError):
        FP8AdamW(p, g, param_bf16=[torch.zeros(100, device=dev)])              # not bf16
    with pytest.raises(ValueError):
        FP8AdamW(p, g, m=[torch.zeros(200, device=dev, dtype=torch.uint8)[::2]])  # not contiguous
    opt = FP8AdamW(p, g, m_fmt="fp32", m=[torch.zeros(100, device=dev)])       # fp32 m in fp32 mode
    opt.step()
    opt.close()
