"""Failure detection without a GPU fault: bad data that only the device can see, and a pipeline
wait that runs out of time. Each sets the per-device error word, which dg_get_device_error()
returns (and clears); the work that is still well-defined is done, and the context stays usable.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import _lib, build, ops, synth
from tests.gpu_util import assert_close, bf16_dev, bf16_host_f64, dev, host

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
MODE = os.environ.get("DG_TEST_SKIP_RELEASE", "")
CHILD = MODE in ("1", "2", "3", "4")


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


@pytest.mark.skipif(CHILD, reason="parent-process test")
def test_contiguous_expert_id_out_of_range(oracle):
    """A 128-row block whose expert id is >= G: the error word says DG_ERR_DEVICE, that block is
    skipped, and every other block is computed as usual."""
    G, N, K = 4, 264, 256
    m, layout, x, w = synth.contiguous_inputs(G, N, K, lo=200, hi=300, salt=31)
    layout = layout.copy()
    bad = 2 * 128                                         # third 128-row block
    assert layout[bad] >= 0
    layout[bad:bad + 128] = G + 1
    a, sfa = ops.cast_per_token(bf16_dev(x))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    assert _lib.dg_get_device_error() == _lib.DG_OK
    d = ops.m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, dev(layout))
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_ERR_DEVICE
    assert _lib.dg_get_device_error() == _lib.DG_OK       # read and cleared
    ok_layout = layout.copy()
    ok_layout[bad:bad + 128] = -1                         # the oracle's view: no expert there
    rows = np.nonzero(ok_layout >= 0)[0].astype(np.int32)
    ref = oracle.m_grouped_contiguous(host(a), host(sfa), host(b), host(sfb), ok_layout, None, rows=rows)
    assert_close(bf16_host_f64(d)[rows], ref, "contiguous with one bad block")


@pytest.mark.skipif(CHILD, reason="parent-process test")
def test_masked_m_above_m_max(oracle):
    """masked_m[g] > M_max: the error word says DG_ERR_DEVICE and the expert is computed as if
    masked_m[g] were M_max."""
    G, M_max, N, K = 3, 160, 264, 256
    masked_m, a_bits, w = synth.masked_inputs(G, M_max, N, K, lo=10, hi=160, salt=32)
    a, sfa = ops.cast_per_token(bf16_dev(a_bits))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    given = masked_m.copy()
    given[1] = M_max + 5
    d = bf16_dev(np.full((G, M_max, N), synth.sentinel_bf16(), np.uint16))
    ops.m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, dev(given), 192, out=d)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_ERR_DEVICE
    clamped = given.copy()
    clamped[1] = M_max
    ref = oracle.m_grouped_masked(host(a), host(sfa), host(b), host(sfb), clamped)
    dh = bf16_host_f64(d)
    for g in range(G):
        assert_close(dh[g, :clamped[g]], ref[g, :clamped[g]], f"masked expert {g}")


@pytest.mark.skipif(CHILD, reason="parent-process test")
def test_pipeline_wait_timeout_is_reported():
    """A child process withholds one TMEM-buffer release in the tile GEMM (a debug-only switch)
    with a 100 ms wait limit: the MMA issuer's wait runs out, the kernel stops and returns, and
    DG_ERR_TIMEOUT is reported; the context then still computes correctly."""
    env = dict(os.environ, DG_TEST_SKIP_RELEASE="1", DG_WAIT_TIMEOUT_MS="100")
    cmd = [sys.executable, "-m", "pytest", os.path.join(HERE, "test_gpu_failure.py"), "-q", "-x", "-m", "gpu",
           "-k", "child"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    assert r.returncode == 0 and " passed" in r.stdout, tail


@pytest.mark.skipif(CHILD, reason="parent-process test")
def test_cluster_exchange_wait_timeout_is_reported():
    """A child process makes one math warp of the first cluster of the cluster split-K kernel
    withhold its partial-push arrive (a debug-only switch), with a 100 ms wait limit: the reducers'
    waits run out, every CTA of the cluster still meets the final cluster barrier and frees TMEM,
    and DG_ERR_TIMEOUT is reported; the context then still computes correctly."""
    env = dict(os.environ, DG_TEST_SKIP_RELEASE="2", DG_WAIT_TIMEOUT_MS="100", DG_FEW_ROW="cluster")
    cmd = [sys.executable, "-m", "pytest", os.path.join(HERE, "test_gpu_failure.py"), "-q", "-x", "-m", "gpu",
           "-k", "child"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    assert r.returncode == 0 and " passed" in r.stdout, tail


@pytest.mark.skipif(MODE != "2", reason="runs in the child process of test_cluster_exchange_wait_timeout_is_reported")
def test_child_cluster_timeout_then_recovery(oracle):
    M, N, K = 64, 2112, 7168                              # 17 tiles: clusters of 6 CTAs
    x, w, c = synth.dense_inputs(M, N, K, False, salt=43)
    a, sfa = ops.cast_per_token(bf16_dev(x))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ops.fp8_gemm_nt(a, sfa, b, sfb, None)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_ERR_TIMEOUT
    assert _lib.dg_get_device_error() == _lib.DG_OK
    # the context is usable: a many-row GEMM (the tile kernel, no withheld arrive) is exact
    M2, N2, K2 = 512, 512, 1024
    x2, w2, _ = synth.dense_inputs(M2, N2, K2, False, salt=44)
    a2, sfa2 = ops.cast_per_token(bf16_dev(x2))
    b2, sfb2 = ops.cast_per_block(bf16_dev(w2))
    d2 = ops.fp8_gemm_nt(a2, sfa2, b2, sfb2, None)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ref = oracle.gemm_nt(host(a2), host(sfa2), host(b2), host(sfb2), None)
    assert_close(bf16_host_f64(d2), ref, "after a cluster timeout")


@pytest.mark.skipif(MODE != "1", reason="runs in the child process of test_pipeline_wait_timeout_is_reported")
def test_child_timeout_then_recovery(oracle):
    M, N, K = 512, 512, 1024                              # CTA-pair tiles, several K blocks
    x, w, c = synth.dense_inputs(M, N, K, False, salt=41)
    a, sfa = ops.cast_per_token(bf16_dev(x))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ops.fp8_gemm_nt(a, sfa, b, sfb, None)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_ERR_TIMEOUT
    assert _lib.dg_get_device_error() == _lib.DG_OK
    # the context is usable: a few-row GEMM (another kernel, no withheld release) is exact
    M2, N2, K2 = 64, 2112, 7168
    x2, w2, _ = synth.dense_inputs(M2, N2, K2, False, salt=42)
    a2, sfa2 = ops.cast_per_token(bf16_dev(x2))
    b2, sfb2 = ops.cast_per_block(bf16_dev(w2))
    d2 = ops.fp8_gemm_nt(a2, sfa2, b2, sfb2, None)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ref = oracle.gemm_nt(host(a2), host(sfa2), host(b2), host(sfb2), None)
    assert_close(bf16_host_f64(d2), ref, "after a timeout")


@pytest.mark.skipif(CHILD, reason="parent-process test")
def test_streamk_flag_wait_timeout_leaves_no_stale_flags():
    """A child process makes the odd-numbered CTAs of its first two stream-K launches withhold
    their partial flags (a debug-only switch), with a 100 ms wait limit: the owners' flag waits
    run out, leaving the flags of the partials they did not reach set. Without a
    dg_get_device_error() call in between, the next stream-K launches on the same per-stream
    workspace and on the static scratch of dg_fp8_gemm_nt_noalloc must still be exact."""
    env = dict(os.environ, DG_TEST_SKIP_RELEASE="3", DG_WAIT_TIMEOUT_MS="100", DG_FEW_ROW="streamk")
    cmd = [sys.executable, "-m", "pytest", os.path.join(HERE, "test_gpu_failure.py"), "-q", "-x", "-m", "gpu",
           "-k", "child"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    assert r.returncode == 0 and " passed" in r.stdout, tail


@pytest.mark.skipif(MODE != "3", reason="runs in the child process of test_streamk_flag_wait_timeout_leaves_no_stale_flags")
def test_child_streamk_timeout_then_exact(oracle):
    M, N, K = 64, 4096, 7168          # 32 weight tiles of 56 K blocks: 4-6 partials per tile
    x, w, c = synth.dense_inputs(M, N, K, True, salt=45)
    x_bad, _, _ = synth.dense_inputs(M, N, K, False, salt=46)
    b, sfb = ops.cast_per_block(bf16_dev(w))
    a, sfa = ops.cast_per_token(bf16_dev(x))
    a_bad, sfa_bad = ops.cast_per_token(bf16_dev(x_bad))   # other partials, so stale ones would show
    cd = bf16_dev(c)
    assert _lib.dg_get_device_error() == _lib.DG_OK

    def out():
        return torch.full((M, N), -3.0, dtype=torch.bfloat16, device="cuda")

    # the two withholding launches: the per-stream workspace, then the static scratch
    _lib.dg_fp8_gemm_nt(a_bad, sfa_bad, b, sfb, cd, out(), M, N, K)
    _lib.dg_fp8_gemm_nt_noalloc(a_bad, sfa_bad, b, sfb, cd, out(), M, N, K)
    # no dg_get_device_error() here: the next launches find the flags as the failed ones left them
    d_ws, d_static = out(), out()
    _lib.dg_fp8_gemm_nt(a, sfa, b, sfb, cd, d_ws, M, N, K)
    _lib.dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, cd, d_static, M, N, K)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_ERR_TIMEOUT
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ref = oracle.gemm_nt(host(a), host(sfa), host(b), host(sfb), c)
    assert_close(bf16_host_f64(d_ws), ref, "stream-K after a flag timeout")
    assert torch.equal(d_static.view(torch.int16), d_ws.view(torch.int16))


@pytest.mark.skipif(CHILD, reason="parent-process test")
def test_tail_flag_wait_timeout_then_exact():
    """A child process makes the piece CTAs of its first last-wave-split tile GEMM withhold their
    partial flags (a debug-only switch), with a 100 ms wait limit: the first pieces' flag waits
    run out and DG_ERR_TIMEOUT is reported; the next launch on the same workspace is exact."""
    env = dict(os.environ, DG_TEST_SKIP_RELEASE="4", DG_WAIT_TIMEOUT_MS="100")
    cmd = [sys.executable, "-m", "pytest", os.path.join(HERE, "test_gpu_failure.py"), "-q", "-x", "-m", "gpu",
           "-k", "child"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    assert r.returncode == 0 and " passed" in r.stdout, tail


@pytest.mark.skipif(MODE != "4", reason="runs in the child process of test_tail_flag_wait_timeout_then_exact")
def test_child_tail_timeout_then_exact(oracle):
    M, N, K = 512, 2048, 7168          # 16 pair tiles, each cut into pieces along K
    x, w, c = synth.dense_inputs(M, N, K, True, salt=47)
    x_bad, _, _ = synth.dense_inputs(M, N, K, False, salt=48)
    b, sfb = ops.cast_per_block(bf16_dev(w))
    a, sfa = ops.cast_per_token(bf16_dev(x))
    a_bad, sfa_bad = ops.cast_per_token(bf16_dev(x_bad))   # other partials, so stale ones would show
    cd = bf16_dev(c)
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ops.fp8_gemm_nt(a_bad, sfa_bad, b, sfb, cd)              # withholds its flags
    assert "last-wave split" in _lib.dg_last_kernel()
    d = ops.fp8_gemm_nt(a, sfa, b, sfb, cd)                 # no dg_get_device_error() in between
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_ERR_TIMEOUT
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ref = oracle.gemm_nt(host(a), host(sfa), host(b), host(sfb), c)
    assert_close(bf16_host_f64(d), ref, "last-wave split after a flag timeout")
