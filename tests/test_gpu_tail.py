"""GPU parity of the dense tile GEMM's last-wave split against the oracle, element by element
within |D - ref| <= 2^-7·|ref| + 1e-2·rms(ref).

When the tiles of a dense GEMM with M > 128 do not fill a whole number of waves of resident
CTAs (pairs), the last wave's tiles are cut along K into pieces that run at once; the CTAs of
the later pieces hand their fp32 partial sums to the first piece's CTA through the stream's
flag workspace, which adds them in piece order and writes D. The shapes below take the split
with no, one or several whole waves before it, on CTA pairs (256-column tiles), single CTAs
(128- and 256-column tiles), ragged rows and columns, with and without C, and piece counts
that do and do not divide the K blocks evenly (a forced count, in a child process).
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import _lib, build, ops, synth
from tests.gpu_util import assert_close, bf16_dev, bf16_host_f64, host

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CHILD = os.environ.get("DG_TAIL_TEST", "")


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def operands(M, N, K, with_c, salt):
    x, w, c = synth.dense_inputs(M, N, K, with_c, salt=salt)
    a, sfa = ops.cast_per_token(bf16_dev(x))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    return (a, sfa, b, sfb, bf16_dev(c) if c is not None else None), c


def check(oracle, M, N, K, with_c, salt, expect_split=True):
    dv, c = operands(M, N, K, with_c, salt)
    a, sfa, b, sfb, cd = dv
    d = ops.fp8_gemm_nt(a, sfa, b, sfb, cd)
    torch.cuda.synchronize()
    name = _lib.dg_last_kernel()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    if expect_split:
        assert "last-wave split" in name, name
    ref = oracle.gemm_nt(host(a), host(sfa), host(b), host(sfb), c)
    assert_close(bf16_host_f64(d), ref, f"{M}x{N}x{K} c={with_c} ({name})")
    return dv, d


# (M, N, K): tiles over 74 resident CTA pairs (148 CTAs for 128-column tiles), and the piece
# count the cost model picks there
AUTO = [
    (512, 2048, 7168, True),    # 16 pair tiles, no whole wave: 4 pieces of 14 K blocks
    (256, 2048, 7168, False),   # 8 pair tiles: 5 pieces of 11 or 12 K blocks
    (4096, 1280, 8192, False),  # 80 pair tiles: one whole wave, then 6 tiles in 5 pieces
    (4096, 128, 8192, True),    # 128-column single-CTA tiles, 32 of them in 4 pieces
    (768, 2112, 7168, True),    # ragged last column block among the split tiles (2 pieces)
    (700, 1000, 7168, False),   # ragged rows and columns (5 pieces)
]


@pytest.mark.skipif(bool(CHILD), reason="parent-process test")
@pytest.mark.parametrize("M,N,K,with_c", AUTO)
def test_tail_split_full_compare(oracle, M, N, K, with_c):
    check(oracle, M, N, K, with_c, salt=M + 3 * N + K)


@pytest.mark.skipif(bool(CHILD), reason="parent-process test")
def test_tail_split_deterministic():
    """Bitwise the same result launch after launch: the partials are added in piece order, and
    a flag left by an earlier launch (an older ticket) is never taken for this launch's."""
    dv, _ = operands(512, 2048, 7168, True, salt=5)
    d1 = ops.fp8_gemm_nt(*dv)
    assert "last-wave split" in _lib.dg_last_kernel()
    for _ in range(4):
        d2 = ops.fp8_gemm_nt(*dv)
        assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))


@pytest.mark.skipif(bool(CHILD), reason="parent-process test")
def test_tail_split_c_aliases_d(oracle):
    """C passed as D: the last-wave pieces read C of their own tiles only, which the launch of the
    whole waves, running beside them, never writes."""
    M, N, K = 4096, 1280, 8192
    dv, c = operands(M, N, K, True, salt=8)
    a, sfa, b, sfb, cd = dv
    d = cd.clone()
    ops.fp8_gemm_nt(a, sfa, b, sfb, d, out=d)
    torch.cuda.synchronize()
    assert "last-wave split" in _lib.dg_last_kernel()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ref = oracle.gemm_nt(host(a), host(sfa), host(b), host(sfb), c)
    assert_close(bf16_host_f64(d), ref, "last-wave split with C aliasing D")


@pytest.mark.skipif(bool(CHILD), reason="parent-process test")
def test_tail_split_under_graph_replay():
    """Captured into a CUDA graph after the stream's workspace exists, the split GEMM replays
    with the launch tickets advancing replay after replay: same bits as the eager call."""
    dv, _ = operands(256, 2048, 7168, True, salt=6)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        d_eager = ops.fp8_gemm_nt(*dv)          # allocates the stream's workspace
        assert "last-wave split" in _lib.dg_last_kernel()
        out = torch.empty_like(d_eager)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            ops.fp8_gemm_nt(*dv, out=out)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), d_eager.view(torch.int16))
    assert _lib.dg_get_device_error() == _lib.DG_OK


def run_child(mode, extra_env):
    env = dict(os.environ, DG_TAIL_TEST=mode, **extra_env)
    cmd = [sys.executable, "-m", "pytest", os.path.join(HERE, "test_gpu_tail.py"), "-q", "-x", "-m", "gpu",
           "-k", "child"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    assert r.returncode == 0 and " passed" in r.stdout, tail


@pytest.mark.skipif(bool(CHILD), reason="parent-process test")
def test_tail_split_forced_pieces():
    """A forced piece count (7: uneven pieces of 4 and 5 K blocks), on CTA pairs and, with pairs
    turned off, on single CTAs with 256-column tiles."""
    run_child("pairs", {"DG_TAIL_SPLIT": "7"})
    run_child("single", {"DG_TAIL_SPLIT": "7", "DG_FORCE_PAIR": "0"})


@pytest.mark.skipif(CHILD not in ("pairs", "single"), reason="runs in a child process")
@pytest.mark.parametrize("M,N,K,with_c", [(512, 1024, 4096, True), (1280, 1536, 3584, False), (4096, 128, 2048, True)])
def test_child_forced_pieces(oracle, M, N, K, with_c):
    check(oracle, M, N, K, with_c, salt=M + N + 11)


@pytest.mark.skipif(bool(CHILD), reason="parent-process test")
def test_tail_split_off_gives_whole_tiles(oracle):
    """DG_TAIL_SPLIT=0: a shape the cost model splits runs its last wave whole instead."""
    run_child("off", {"DG_TAIL_SPLIT": "0"})


@pytest.mark.skipif(CHILD != "off", reason="runs in a child process")
def test_child_split_off(oracle):
    check(oracle, 512, 2048, 7168, True, salt=21, expect_split=False)
    assert "last-wave split" not in _lib.dg_last_kernel()
