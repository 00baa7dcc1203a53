"""The opt-in bf16 GEMM kernels against the oracle.

The library picks its expert GEMM kernel once per process from MOE_BF16_GEMM
("dual": two token tiles per weight tile, "pair": CTA pairs); the default
one-tile kernel is covered by the other GPU tests.  Each variant reruns the
bf16 layer parity tests (routing and dispatch bit-exact, expert outputs and
the layer within the bf16 tolerance) in a child process with the variable set.
Likewise MOE_WGRAD=single selects the one-CTA weight-gradient kernel instead
of the default CTA-pair one; the weight-gradient parity tests rerun with it.
MOE_FP8_EPI picks the FP8 GEMM epilogue's TMEM read shape (narrow, x32,
wide32; the default is the eight-warp one); the FP8 layer and FP8
input-gradient parity tests rerun with each.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", ["dual", "pair"])
def test_bf16_expert_gemm_variant(kind):
    env = dict(os.environ, MOE_BF16_GEMM=kind)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(HERE, "test_gpu_parity.py"),
           "-k", "small_bf16 or mid_bf16 or all_experts or idle"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail


def test_one_cta_weight_gradient_kernel():
    env = dict(os.environ, MOE_WGRAD="single")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(HERE, "test_gpu_backward.py"), "-k", "dw"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail


@pytest.mark.parametrize("kind", ["narrow", "x32", "wide32"])
def test_fp8_epilogue_variant(kind):
    env = dict(os.environ, MOE_FP8_EPI=kind)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(HERE, "test_gpu_parity.py"), os.path.join(HERE, "test_gpu_fp8_backward.py"),
           "-k", "small_fp8 or backward_dx"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail


def test_fp8_dispatch_direct_scales():
    """MOE_FP8_SCALES=direct: the dispatch writes its E4M3 scales straight to
    the block-major array instead of staging them per row; the FP8 layer
    parity tests (codes and scales bit-exact) rerun with it."""
    env = dict(os.environ, MOE_FP8_SCALES="direct")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(HERE, "test_gpu_parity.py"), "-k", "small_fp8"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail


@pytest.mark.parametrize("kind", ["wide", "narrow"])
def test_fp8_weight_gradient_shapes(kind):
    """MOE_FP8_WGRAD_EPI: the FP8 weight-gradient kernel on 256-column tiles
    (eight or sixteen epilogue warps) instead of the default 128-column tiles;
    the FP8 weight-gradient parity test reruns with each."""
    env = dict(os.environ, MOE_FP8_WGRAD_EPI=kind)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(HERE, "test_gpu_fp8_backward.py"), "-k", "dw"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail
