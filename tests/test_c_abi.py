"""The library from plain C: tests/c_abi_example.c includes only
include/fp8adam.h and the CUDA runtime header, links libfp8adam.so, and runs
steps through fp8adam_create / fp8adam_step / fp8adam_check.  On CPU it must
compile (as C11, warnings as errors) and link; on a GPU its results must equal
the oracle's bit for bit."""
import os
import subprocess

import numpy as np
import pytest
import torch

from fp8_quantized_adam_b200 import build as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(tmp_path) -> str:
    b.build()
    exe = str(tmp_path / "c_abi_example")
    lib_dir = os.path.dirname(b.LIB)
    cmd = ["gcc", "-std=c11", "-O1", "-Wall", "-Wextra", "-Werror", os.path.join(ROOT, "tests", "c_abi_example.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"), "-L", lib_dir, "-lfp8adam",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + lib_dir,
           "-Wl,-rpath," + os.path.join(CUDA, "lib64"), "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_example_compiles_and_links(tmp_path):
    assert os.path.exists(_compile(tmp_path))


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.gpu
def test_c_example_matches_the_oracle(tmp_path):
    import oracle

    exe = _compile(tmp_path)
    rng = np.random.default_rng(71)
    sizes = [70001, 4097]
    steps = 4
    p0 = [(rng.standard_normal(n) * 0.02).astype(np.float32) for n in sizes]
    grads = [[_bf16_bits(rng.standard_normal(n) * 10.0 ** rng.uniform(-6, -1, n)) for n in sizes]
             for _ in range(steps)]
    inp, outp = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(inp, "wb") as f:
        f.write(np.array(sizes, np.int64).tobytes())
        for p in p0:
            f.write(p.tobytes())
        for gs in grads:
            for g in gs:
                f.write(g.tobytes())
    r = subprocess.run([exe, str(inp), str(outp), str(steps)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, (r.returncode, r.stderr)

    ref = [oracle.TensorState(p, oracle.E4M3, oracle.E5M2) for p in p0]
    for t in range(1, steps + 1):
        for i, st in enumerate(ref):
            st.step(grads[t - 1][i], 3e-4, 0.9, 0.95, 1e-8, 0.1, t)
    data = outp.read_bytes()
    off = 0
    for i, n in enumerate(sizes):
        p = np.frombuffer(data, np.uint32, n, off)
        off += 4 * n
        m = np.frombuffer(data, np.uint8, n, off)
        off += n
        v = np.frombuffer(data, np.uint8, n, off)
        off += n
        assert (p == ref[i].p.view(np.uint32)).all(), i
        assert (m == ref[i].m).all() and (v == ref[i].v).all(), i
    state = np.frombuffer(data, np.float32, 8, off)
    for i in range(2):
        assert state[0 + i] == ref[i].scale_m[0] and state[2 + i] == ref[i].scale_v[0]
        assert state[4 + i] == ref[i].amax_m[0] and state[6 + i] == ref[i].amax_v[0]


def test_header_compiles_as_cpp(tmp_path):
    """The header's extern "C" guard: a C++ translation unit sees C linkage."""
    src = tmp_path / "use.cpp"
    src.write_text('#include "fp8adam.h"\n'
                   'extern "C" int fp8adam_step(fp8adam_ctx*, float, float, float, float, float, int64_t, void*);\n'
                   'int main() { return fp8adam_strerror(FP8ADAM_OK) ? 0 : 1; }\n')
    r = subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-I",
                        os.path.join(ROOT, "include"), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
