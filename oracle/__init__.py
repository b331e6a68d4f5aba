"""CPU oracle (test infrastructure, not product code).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg import this package.  It shares no code with the CUDA library.  Every
function is pinned by ``tests/test_oracle_pins.py``; no function is "parity
unpinned".
"""
from .fp8_gemm import (  # noqa: F401
    BLOCK,
    bf16_bits_from_f64,
    bf16_bits_to_f64,
    e4m3_table,
    fp8_gemm_nt,
    fp8_gemm_nt_f64,
    m_grouped_fp8_gemm_nt_contiguous,
    m_grouped_fp8_gemm_nt_masked,
    pack_sf_ue8m0,
    packed_sf_shape,
    ue8m0_from_f32,
    ue8m0_value,
    unpack_sf_ue8m0,
)
