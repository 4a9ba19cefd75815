"""Parity of the kernel choices the default dispatch does not take for the test shapes.

The library picks GEMM kernels by shape: for few-row dense problems a swapped-operand kernel,
either the cluster split-K one (few tiles, moderate K) or the stream-K one, and the CTA-pair
kernel for everything else, the masked MoE layout included. Each choice can be forced per
process through environment variables, which the library reads once (``DG_FORCE_SWAP``,
``DG_FEW_ROW``, ``DG_SPLITK_S`` for the cluster size, ``DG_FORCE_PAIR``). Each test below re-runs a
selection of the parity tests in a child pytest process with overrides set, so that every
kernel variant is compared with the oracle on the same cases.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

CASES = [
    # (environment, test file, -k selection)
    ({"DG_FORCE_SWAP": "1"}, "test_gpu_grouped.py", "masked_small or masked_edge or masked_page"),
    ({"DG_FORCE_SWAP": "1", "DG_FEW_ROW": "cluster"}, "test_gpu_grouped.py", "masked_small or masked_edge or masked_page"),
    ({"DG_FORCE_SWAP": "0"}, "test_gpu_gemm.py", "decode or small"),
    ({"DG_FEW_ROW": "streamk"}, "test_gpu_gemm.py", "decode or small or repeatable"),
    ({"DG_FEW_ROW": "cluster"}, "test_gpu_gemm.py", "decode or small or repeatable"),
    ({"DG_FEW_ROW": "cluster", "DG_SPLITK_S": "1"}, "test_gpu_gemm.py", "small or repeatable"),
    ({"DG_FEW_ROW": "cluster", "DG_SPLITK_S": "2"}, "test_gpu_gemm.py", "small or repeatable"),
    ({"DG_FEW_ROW": "cluster", "DG_SPLITK_S": "3"}, "test_gpu_gemm.py", "small or repeatable"),
    ({"DG_FEW_ROW": "cluster", "DG_SPLITK_S": "6"}, "test_gpu_gemm.py", "small or repeatable"),
    ({"DG_FEW_ROW": "cluster", "DG_SPLITK_S": "8"}, "test_gpu_gemm.py", "small or repeatable"),
    ({"DG_FEW_ROW": "cluster", "DG_SPLITK_S": "16"}, "test_gpu_gemm.py", "small or repeatable"),
    ({"DG_FORCE_PAIR": "0"}, "test_gpu_grouped.py", "masked_small or masked_edge or contiguous_small"),
    ({"DG_FORCE_PAIR": "0"}, "test_gpu_gemm.py", "small or repeatable"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("env,path,select", CASES, ids=["-".join(f"{k}={v}" for k, v in e.items()) + f"-{p[9:-3]}"
                                                      for e, p, _ in CASES])
def test_forced_kernel_parity(env, path, select):
    child_env = dict(os.environ)
    child_env.update(env)
    cmd = [sys.executable, "-m", "pytest", os.path.join(HERE, path), "-q", "-x", "-m", "gpu", "-k", select]
    r = subprocess.run(cmd, cwd=ROOT, env=child_env, capture_output=True, text=True, timeout=1800)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    assert r.returncode == 0, f"{env} {path} -k '{select}' failed:\n{tail}"
    assert " passed" in r.stdout, f"nothing ran for {env} {path} -k '{select}':\n{tail}"
