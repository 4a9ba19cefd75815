"""B200 (sm_100a) FP8 block-scaled NT GEMM: dense, M-grouped contiguous and masked MoE
variants, the FP8 cast-and-scale kernels and the scale-layout transform.

The compute lives in ``libdg_b200.so`` (CUDA, built by ``python -m moe_grouped_gemm_sm_b200.build``)
behind the C ABI of ``include/dg.h``; :mod:`moe_grouped_gemm_sm_b200._lib` binds it with the
same names, and :mod:`moe_grouped_gemm_sm_b200.ops` adds torch-tensor conveniences that only
allocate outputs and marshal arguments. :mod:`moe_grouped_gemm_sm_b200.synth` draws the
seeded synthetic workloads.
"""
from ._lib import (DgError, dg_cast_fp8_per_block, dg_cast_fp8_per_token, dg_fp8_gemm_nt,  # noqa: F401
                   dg_get_device_error, dg_m_grouped_fp8_gemm_nt_contiguous, dg_m_grouped_fp8_gemm_nt_masked,
                   dg_sf_ld, dg_status_string, dg_transform_sf)

__version__ = "0.1.0"
