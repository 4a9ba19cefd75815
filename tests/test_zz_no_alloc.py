"""dg_fp8_gemm_nt_noalloc: the stream-K few-row GEMM with the library's static scratch instead of
the per-stream workspace. It must give exactly what dg_fp8_gemm_nt gives when that call takes
the stream-K kernel too (same kernel, same work split), call after call (flags left set by an
earlier launch never match a later launch's ticket), allocate no device memory, work under
CUDA-graph capture on a fresh stream, and refuse rows it cannot take. Some callers cannot
allocate at all: a runtime that owns every byte of device memory through its own arena, or a
decode loop whose memory plan is fixed; this entry point serves them.

dg_fp8_gemm_nt picks its few-row kernel by shape; DG_FEW_ROW=streamk makes it always take the
stream-K kernel. The library reads that variable once per process, so the tests that compare
with dg_fp8_gemm_nt run in a child pytest process with it set."""
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
CHILD = os.environ.get("DG_FEW_ROW") == "streamk"
child_only = pytest.mark.skipif(not CHILD, reason="runs in the DG_FEW_ROW=streamk child process")


@pytest.mark.skipif(CHILD, reason="parent-process test")
def test_in_a_streamk_child_process():
    env = dict(os.environ, DG_FEW_ROW="streamk")
    cmd = [sys.executable, "-m", "pytest", os.path.join(HERE, "test_zz_no_alloc.py"), "-q", "-x", "-m", "gpu"]
    r = subprocess.run(cmd, cwd=os.path.dirname(HERE), env=env, capture_output=True, text=True, timeout=1200)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    assert r.returncode == 0 and " passed" in r.stdout, tail

SHAPES = [(1, 128, 128), (37, 264, 640), (64, 2112, 7168), (100, 1000, 896), (128, 4096, 7168)]


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def operands(M, N, K, with_c, salt):
    x, w, c = synth.dense_inputs(M, N, K, with_c, salt=salt)
    a, sfa = ops.cast_per_token(bf16_dev(x))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    cd = bf16_dev(c) if c is not None else None
    return (a, sfa, b, sfb, cd), (x, w, c)


def sentinel(M, N):
    return torch.full((M, N), -3.0, dtype=torch.bfloat16, device="cuda")


@child_only
@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("with_c", [False, True])
def test_same_bits_as_the_allocating_entry_point_twice(M, N, K, with_c):
    (a, sfa, b, sfb, c), _ = operands(M, N, K, with_c, salt=M + N + K)
    ref = sentinel(M, N)
    _lib.dg_fp8_gemm_nt(a, sfa, b, sfb, c, ref, M, N, K)
    outs = []
    for _ in range(2):                       # the second call finds the flags the first left
        d = sentinel(M, N)
        _lib.dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, c, d, M, N, K)
        outs.append(d)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    for d in outs:
        assert torch.equal(d.view(torch.int16), ref.view(torch.int16))


def test_matches_the_oracle(oracle):
    M, N, K = 64, 2112, 7168
    (a, sfa, b, sfb, c), (x, w, cb) = operands(M, N, K, True, salt=5)
    d = sentinel(M, N)
    _lib.dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, c, d, M, N, K)
    torch.cuda.synchronize()
    ref = oracle.gemm_nt(host(a), host(sfa), host(b), host(sfb), cb)
    assert_close(bf16_host_f64(d), ref, "noalloc 64x2112x7168")


@child_only
def test_allocates_nothing_on_a_new_stream():
    """The library counts every byte it allocates (dg_allocated_bytes): a call on a stream that
    never saw one leaves the count as it was, where dg_fp8_gemm_nt allocates that stream's
    workspace."""
    M, N, K = 64, 2112, 7168
    (a, sfa, b, sfb, c), _ = operands(M, N, K, True, salt=6)
    d = sentinel(M, N)
    _lib.dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, c, d, M, N, K)   # kernel loaded, tensors ready
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    before = _lib.dg_allocated_bytes()
    torch_before = torch.cuda.memory_allocated()
    _lib.dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, c, d, M, N, K, stream=s)
    torch.cuda.synchronize()
    assert _lib.dg_allocated_bytes() == before
    assert torch.cuda.memory_allocated() == torch_before
    # the allocating entry point does allocate its workspace for a new stream
    s2 = torch.cuda.Stream()
    _lib.dg_fp8_gemm_nt(a, sfa, b, sfb, c, d, M, N, K, stream=s2)
    torch.cuda.synchronize()
    assert _lib.dg_allocated_bytes() > before


@child_only
def test_graph_capture_on_a_fresh_stream_replays_exactly():
    M, N, K = 64, 2112, 7168
    (a, sfa, b, sfb, c), _ = operands(M, N, K, False, salt=7)
    eager = sentinel(M, N)
    _lib.dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, c, eager, M, N, K)
    torch.cuda.synchronize()
    d = sentinel(M, N)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        _lib.dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, c, d, M, N, K, stream=s)
    for _ in range(3):
        d.fill_(-3.0)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(d.view(torch.int16), eager.view(torch.int16))
    assert _lib.dg_get_device_error() == _lib.DG_OK


def test_refuses_more_than_128_rows():
    M, N, K = 129, 256, 256
    (a, sfa, b, sfb, c), _ = operands(M, N, K, False, salt=8)
    d = sentinel(M, N)
    with pytest.raises(_lib.DgError) as e:
        _lib.dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, c, d, M, N, K)
    assert e.value.status == _lib.DG_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((d == -3.0).all())
