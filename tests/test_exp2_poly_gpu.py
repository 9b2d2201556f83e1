"""The FMA-pipe exponentials of the attention kernels, tested on their own.

The softmax of both attention kernels evaluates a share of its 2^x on the FMA
pipe instead of the MUFU unit (``csrc/sm100_ptx.cuh``): a Cody–Waite split
x = j + r with |r| <= 1/2, a polynomial for 2^r, and j added to the exponent
field.  ``exp2_poly2`` (cubic) serves bf16 P, ``exp2_poly2q`` (quadratic) the
e4m3 P of the 8-bit kernel.  Their stated properties, checked here on a dense
grid against 2^x evaluated in fp64 on the host:
  * relative error at most 7.5e-5 (cubic) and 1.73e-3 (quadratic) for x in
    [-125, 9] (the kernels' arguments lie in [-125, 8.5]; bf16 P needs 2^-9,
    e4m3 P 2^-4);
  * x below -125 is clamped: the result is 2^-125, a normal float;
  * every result is a finite, normal, positive float.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gpu_probes", "exp2_probe.cu")
CSRC = os.path.join(os.path.dirname(HERE), "diffusion_transformer_attention_attn_b200", "csrc")
LIB = os.path.join(HERE, "gpu_probes", "libexp2_probe.so")
MAX_REL = {0: 7.5e-5, 1: 1.73e-3}   # cubic, quadratic


@pytest.fixture(scope="module")
def probe():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from diffusion_transformer_attention_attn_b200 import build_lib
    header = os.path.join(CSRC, "sm100_ptx.cuh")
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(SRC), os.path.getmtime(header)):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call([build_lib.nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                               "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I", CSRC, SRC, "-o", tmp])
        os.replace(tmp, LIB)
    lib = ctypes.CDLL(LIB)
    lib.exp2_poly_probe.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p]
    lib.exp2_poly_probe.restype = ctypes.c_int
    return lib


def _run(lib, x: np.ndarray, quadratic: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(0.0))
    xd = torch.from_numpy(x).cuda()
    yd = torch.full_like(xd, float("nan"))
    st = lib.exp2_poly_probe(xd.data_ptr(), yd.data_ptr(), x.size // 2, quadratic,
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, st
    torch.cuda.synchronize()
    return yd.cpu().numpy()


@pytest.mark.parametrize("quadratic", [0, 1], ids=["cubic", "quadratic"])
def test_relative_error_bound_on_a_dense_grid(probe, quadratic):
    # every float step of 2^-12 over [-125, 9], plus the half-integers (the
    # ends of the reduced interval) and values just beside them
    grid = np.arange(-125.0, 9.0, 2.0 ** -12)
    halves = np.arange(-125.0, 9.0, 0.5)
    beside = np.concatenate([np.nextafter(halves.astype(np.float32), np.float32(-200)),
                             np.nextafter(halves.astype(np.float32), np.float32(200))])
    x = np.concatenate([grid.astype(np.float32), halves.astype(np.float32), beside])
    y = _run(probe, x, quadratic)[:x.size]
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y.astype(np.float64) - ref) / ref
    worst = int(np.argmax(rel))
    assert rel.max() <= MAX_REL[quadratic], f"max relative error {rel.max():.3e} at x = {x[worst]!r}"
    assert np.isfinite(y).all() and (y >= np.finfo(np.float32).tiny).all()


@pytest.mark.parametrize("quadratic", [0, 1], ids=["cubic", "quadratic"])
def test_clamp_below_minus_125(probe, quadratic):
    x = np.array([-125.0, -125.5, -126.0, -140.0, -1e4, -3.0e38, -np.inf], dtype=np.float32)
    y = _run(probe, x, quadratic)[:x.size]
    tiny = np.float64(2.0) ** -125
    for v in y:
        assert abs(float(v) - tiny) <= MAX_REL[quadratic] * tiny, y
    assert (y >= np.finfo(np.float32).tiny).all()


@pytest.mark.parametrize("quadratic", [0, 1], ids=["cubic", "quadratic"])
def test_integers_within_the_fit(probe, quadratic):
    # at r = 0 the polynomial gives its constant term: 2^j times (1 + its error)
    x = np.arange(-125, 9, dtype=np.float32)
    y = _run(probe, x, quadratic)[:x.size].astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert (np.abs(y - ref) / ref <= MAX_REL[quadratic]).all()
