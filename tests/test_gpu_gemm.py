"""GPU parity of the dense FP8 block-scaled NT GEMM against the oracle, element by element,
within |D - ref| <= 2^-7·|ref| + 1e-2·rms(ref). Operands come from the CUDA casts, which are
checked bit-exact against the oracle casts first, so both sides see the same e4m3 codes and
scales."""
import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import build, ops, synth
from tests.gpu_util import assert_close, bf16_dev, bf16_host_f64, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def quantised(oracle, M, N, K, with_c, salt):
    x, w, c = synth.dense_inputs(M, N, K, with_c, salt=salt)
    a, sfa = ops.cast_per_token(bf16_dev(x))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    ao, sfao = oracle.cast_per_token(x)
    bo, sfbo = oracle.cast_per_block(w)
    assert np.array_equal(host(a), ao) and np.array_equal(host(b), bo)
    assert np.array_equal(host(sfa), sfao) and np.array_equal(host(sfb), sfbo)
    return (a, sfa, b, sfb, bf16_dev(c) if c is not None else None), (ao, sfao, bo, sfbo, c)


SMALL = [
    (1, 128, 128), (63, 264, 256), (64, 128, 384), (65, 2112, 256), (127, 136, 512), (129, 520, 128),
    (300, 384, 640), (256, 256, 1024), (200, 8, 256), (130, 1000, 896), (512, 2304, 256),
]


@pytest.mark.parametrize("M,N,K", SMALL)
@pytest.mark.parametrize("with_c", [False, True])
def test_dense_small_full_compare(oracle, M, N, K, with_c):
    dv, hv = quantised(oracle, M, N, K, with_c, salt=M * 7 + N + K)
    a, sfa, b, sfb, c = dv
    d = ops.fp8_gemm_nt(a, sfa, b, sfb, c)
    torch.cuda.synchronize()
    ref = oracle.gemm_nt(*hv)
    assert_close(bf16_host_f64(d), ref, f"{M}x{N}x{K} c={with_c}")


@pytest.mark.parametrize("M,N,K", [(512, 10240, 256), (400, 10176, 384)])
def test_dense_partial_last_wave(oracle, M, N, K):
    """More 256 x 256 pair tiles than one wave of resident CTA pairs, the last wave partial,
    with ragged rows and columns."""
    dv, hv = quantised(oracle, M, N, K, True, salt=M + N)
    a, sfa, b, sfb, c = dv
    d = ops.fp8_gemm_nt(a, sfa, b, sfb, c)
    torch.cuda.synchronize()
    assert_close(bf16_host_f64(d), oracle.gemm_nt(*hv), f"{M}x{N}x{K} last wave")


def test_dense_c_aliases_d(oracle):
    M, N, K = 192, 384, 512
    dv, hv = quantised(oracle, M, N, K, True, salt=9)
    a, sfa, b, sfb, c = dv
    d = c.clone()
    ops.fp8_gemm_nt(a, sfa, b, sfb, d, out=d)
    assert_close(bf16_host_f64(d), oracle.gemm_nt(*hv), "c aliases d")


@pytest.mark.parametrize("M,N,K", [(300, 520, 1024), (64, 2112, 7168), (100, 1000, 896), (128, 24576, 1536)])
def test_dense_repeatable_and_deterministic(oracle, M, N, K):
    """Bitwise the same result, launch after launch: the reductions have a fixed order, and a
    race on a shared-memory ring (a slot refilled while still being read) shows up as runs that
    differ. 128x24576x1536 runs every SM through several tiles."""
    dv, _ = quantised(oracle, M, N, K, True, salt=3)
    d1 = ops.fp8_gemm_nt(*dv)
    for _ in range(4):
        d2 = ops.fp8_gemm_nt(*dv)
        assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))


PAGE_SHAPES = [(2112, 7168), (24576, 1536), (32768, 512), (7168, 16384), (4096, 7168), (7168, 2048)]


def sample_rows(M, per_tile=2, extra=16, seed=0):
    """First and last row of every 128-row tile plus seeded random rows."""
    rows = set()
    for t in range(0, M, 128):
        rows.add(t)
        rows.add(min(M, t + 128) - 1)
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, M, extra).tolist())
    return np.array(sorted(rows), np.int32)


@pytest.mark.slow
@pytest.mark.parametrize("M", [64, 128])
@pytest.mark.parametrize("N,K", PAGE_SHAPES)
def test_decode_shapes_full_compare(oracle, M, N, K):
    """Every element of the twelve decode shapes (at most ~15 G multiply-adds of fp64 on the
    host each). In the few-row kernels the token rows are the MMA's N columns, spread over
    several math warps and, for the split kernels, over several SMs: a fault confined to some
    token columns shows up only in a full compare."""
    with_c = not (M == 64 and (N, K) == (2112, 7168))      # the 64x2112x7168 case has C = 0
    dv, hv = quantised(oracle, M, N, K, with_c, salt=N + K + M)
    d = ops.fp8_gemm_nt(*dv)
    torch.cuda.synchronize()
    ref = oracle.gemm_nt(*hv)
    assert_close(bf16_host_f64(d), ref, f"decode {M}x{N}x{K}")


@pytest.mark.slow
@pytest.mark.parametrize("N,K", PAGE_SHAPES)
def test_prefill_shapes_sampled_rows(oracle, N, K):
    M = 4096
    dv, hv = quantised(oracle, M, N, K, True, salt=N + K)
    d = ops.fp8_gemm_nt(*dv)
    torch.cuda.synchronize()
    rows = sample_rows(M, extra=16, seed=N * 7 + K)
    if N * K > 64 * 2 ** 20:
        rows = rows[::2]
    ref = oracle.gemm_nt(*hv, rows=rows)
    assert_close(bf16_host_f64(d)[rows], ref, f"prefill 4096x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(64, 2112, 7168), (128, 4096, 7168), (64, 24576, 1536)])
def test_few_row_graph_capture_on_a_fresh_stream(oracle, M, N, K):
    """A few-row GEMM captured into a CUDA graph on a stream that never ran one before. The
    cluster split-K shapes (the first two) need no workspace and replay bit for bit what the
    eager call gives. The stream-K shape cannot allocate its workspace under capture and takes
    the tile kernel instead; it replays exactly and stays within the oracle's bound."""
    dv, hv = quantised(oracle, M, N, K, True, salt=M + N)
    eager = ops.fp8_gemm_nt(*dv)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    out = torch.full((M, N), -3.0, dtype=torch.bfloat16, device="cuda")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ops.fp8_gemm_nt(*dv, out=out, stream=s)
    replays = []
    for _ in range(3):
        out.fill_(-3.0)
        g.replay()
        torch.cuda.synchronize()
        replays.append(out.clone())
    for r in replays[1:]:
        assert torch.equal(r.view(torch.int16), replays[0].view(torch.int16))
    cluster_shape = (N + 127) // 128 <= 64 and K // 128 <= 64
    if cluster_shape:
        assert torch.equal(replays[0].view(torch.int16), eager.view(torch.int16))
    ref = oracle.gemm_nt(*hv)
    assert_close(bf16_host_f64(replays[0]), ref, f"graph-captured {M}x{N}x{K}")
