"""The C-ABI library loads, exports every declared entry point, and rejects
bad arguments on the host before touching the GPU (runs without a GPU)."""
import ctypes
import subprocess

import pytest

from moe_grouped_gemm_05_b200 import binding, build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def test_exports_every_declared_symbol(lib):
    names = binding.header_functions()
    assert "dg_fp8_gemm_nt" in names and "dg_pack_sf_ue8m0" in names
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib, n)


def test_pure_host_queries(lib):
    assert lib.dg_get_mk_alignment_for_contiguous_layout() == 128
    assert lib.dg_packed_sf_words(4096, 16) == 4 * 4096
    assert lib.dg_packed_sf_words(56, 16) == 4 * 56
    assert lib.dg_packed_sf_words(13, 7) == 2 * 16
    assert lib.dg_packed_sf_words(-1, 3) == -1


P = ctypes.c_void_p
GOOD = P(0x10000)


def _dense(lib, a=GOOD, sfa=GOOD, b=GOOD, sfb=GOOD, d=GOOD, M=128, N=256, K=256):
    return lib.dg_fp8_gemm_nt(a, sfa, b, sfb, d, M, N, K, None)


def test_dense_argument_errors(lib):
    assert _dense(lib, a=P(0)) == -1
    assert b"non-NULL" in lib.dg_get_last_error()
    assert _dense(lib, b=P(0x10008)) == -3
    assert _dense(lib, K=100) == -2
    assert b"K=100" in lib.dg_get_last_error()
    assert _dense(lib, K=0) == -2
    assert _dense(lib, N=200) == -2
    assert _dense(lib, M=-5) == -2
    assert _dense(lib, M=0) == 0  # empty problem: nothing to do, nothing launched


def test_grouped_argument_errors(lib):
    f = lib.dg_m_grouped_fp8_gemm_nt_contiguous
    assert f(GOOD, GOOD, GOOD, GOOD, GOOD, P(0), 256, 256, 256, 4, None) == -1
    assert f(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 200, 256, 256, 4, None) == -2
    assert f(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 256, 256, 256, 0, None) == -2
    assert f(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 0, 256, 256, 4, None) == 0
    g = lib.dg_m_grouped_fp8_gemm_nt_masked
    assert g(GOOD, GOOD, GOOD, GOOD, GOOD, P(0), 4, 256, 256, 256, None) == -1
    assert g(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 0, 256, 256, 256, None) == -2
    assert g(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 100000, 256, 256, 256, None) == -2
    assert g(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 4, 256, 256, 384 + 1, None) == -2
    assert g(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 4, 0, 256, 256, None) == 0


def test_pack_argument_errors(lib):
    f = lib.dg_pack_sf_ue8m0
    assert f(P(0), GOOD, 1, 4, 4, None) == -1
    assert f(GOOD, P(0x10004), 1, 4, 4, None) == -3
    assert f(GOOD, GOOD, -1, 4, 4, None) == -2
    assert f(GOOD, GOOD, 0, 4, 4, None) == 0


def test_config_override(lib):
    assert lib.dg_set_config(96, 0, 0) == -4
    assert lib.dg_set_config(128, 3, 0) == -4
    assert lib.dg_set_config(256, 0, 2) == -4   # two pipelines: 128- and 224-wide 2-CTA tiles only
    assert lib.dg_set_config(224, 1, 2) == -4
    assert lib.dg_set_config(128, 0, 0) == 0
    assert lib.dg_set_config(224, 2, 0) == 0
    assert lib.dg_set_config(224, 2, 2) == 0
    assert lib.dg_set_config(0, 0, 0) == 0


def test_wait_limit_knob(lib):
    """The pipeline-wait limit is process-wide host state: the setter returns
    the previous value, and the default is 2 s."""
    prev = binding.set_wait_limit_ns(0)
    assert prev == 2_000_000_000
    assert binding.set_wait_limit_ns(123) == 0
    assert binding.set_wait_limit_ns(prev) == 123
    with pytest.raises(ValueError):
        binding.set_wait_limit_ns(-1)


def test_forced_tile_falls_back_per_entry_point(lib):
    """A forced tile that one entry point does not build leaves that entry
    point on the heuristic instead of failing its calls."""
    from moe_grouped_gemm_05_b200 import binding as dg

    heur = dg.describe_config("contiguous", 32768, 4096, 7168, 8)
    assert lib.dg_set_config(64, 1, 1) == 0      # built for dense / masked only
    try:
        assert dg.describe_config("contiguous", 32768, 4096, 7168, 8) == heur
        assert dg.describe_config("dense", 4096, 7168, 2048).startswith("128x64x")
    finally:
        assert lib.dg_set_config(0, 0, 0) == 0


def test_heuristic_choices_without_gpu(lib):
    """The configuration heuristic is host logic: without a device it assumes
    148 SMs.  Decode-sized dense problems take split-K tiles over two
    pipelines, large ones 2-CTA tiles with two pipelines, masked problems
    1-CTA tiles, and the pick is stable for the workloads the bench times."""
    from moe_grouped_gemm_05_b200 import binding as dg

    # at most 64 rows: split-K tiles whose stages hold 64 rows of A
    assert dg.describe_config("dense", 64, 7168, 2048) == "128x64x12(2pipe)(splitk)(a64)/112"
    assert dg.describe_config("dense", 1, 7168, 2048) == "128x64x12(2pipe)(splitk)(a64)/112"
    assert dg.describe_config("dense", 65, 7168, 2048) == "128x64x8(2pipe)(splitk)/112"
    assert dg.describe_config("masked", 64, 256, 2048, 4) == "128x64x10(2pipe)(splitk)(a64)/16"
    assert dg.describe_config("masked", 65, 256, 2048, 4) == "128x64x6(2pipe)(splitk)/16"
    assert lib.dg_set_config(64, 1, 2) == 0  # a forced tile takes the 64-row stages where they fit
    try:
        assert dg.describe_config("dense", 64, 464, 2048).endswith("(a64)/8")
        assert "(a64)" not in dg.describe_config("dense", 65, 464, 2048)
    finally:
        assert lib.dg_set_config(0, 0, 0) == 0
    assert dg.describe_config("dense", 4096, 7168, 2048) == "256x224x6(2cta)(2pipe)/148"
    assert dg.describe_config("dense", 8192, 8192, 8192) == "256x224x6(2cta)(2pipe)/148"
    assert dg.describe_config("dense", 64, 7168, 512) == "128x64x8/112"  # one K group: no split
    masked = dg.describe_config("masked", 256, 7168, 2048, 16)
    assert "(2cta)" not in masked and masked.startswith("128x")
    assert dg.describe_config("contiguous", 32768, 4096, 7168, 8) == "256x224x6(2cta)(2pipe)/148"
    # beyond the pair table's 1024 blocks the contiguous layout keeps 1-CTA tiles
    assert "(2cta)" not in dg.describe_config("contiguous", 1024 * 128 + 128, 4096, 7168, 8)


def test_tc_util_caps_the_planned_grid(lib):
    from moe_grouped_gemm_05_b200 import binding as dg

    assert lib.dg_set_tc_util(0) == -2 and lib.dg_set_tc_util(101) == -2
    assert dg.set_tc_util(50) == 100
    try:
        desc = dg.describe_config("dense", 4096, 7168, 2048)
        assert int(desc.split("/")[-1]) <= 74, desc
    finally:
        assert dg.set_tc_util(100) == 50
    assert dg.describe_config("dense", 4096, 7168, 2048).endswith("/148")


def test_binding_argument_helpers_without_gpu():
    """The binding's checks that keep a wrongly sized tensor from reaching a
    kernel: packed scale element counts, one device for all operands, and
    caller-provided outputs."""
    import torch

    from moe_grouped_gemm_05_b200 import binding as dg

    # [kp, mn4] or [batch, kp, mn4]: ceil(5/4) = 2, align4(5) = 8
    dg._packed_numel(torch.empty(2, 8, dtype=torch.int32), 1, 5, 5, "sfa")
    dg._packed_numel(torch.empty(3, 2, 8, dtype=torch.int32), 3, 5, 5, "sfb")
    with pytest.raises(ValueError, match="expected 3 x 2 x 8"):
        dg._packed_numel(torch.empty(2, 8, dtype=torch.int32), 3, 5, 5, "sfb")
    with pytest.raises(ValueError):
        dg._packed_numel(torch.empty(1, 8, dtype=torch.int32), 1, 5, 5, "sfa")   # one K word short

    x = torch.empty(4)
    dg._same_device(x, torch.empty(2), None)
    from types import SimpleNamespace
    other = SimpleNamespace(get_device=lambda: 1, device="cuda:1")   # stands in for a tensor on GPU 1
    with pytest.raises(ValueError, match="cuda:1"):
        dg._same_device(x, torch.empty(2), other)

    out = torch.empty(3, 4, dtype=torch.bfloat16)
    dg._out(out, (torch.bfloat16,), (3, 4), "out", out.device)
    with pytest.raises(ValueError):
        dg._out(out, (torch.float32,), (3, 4), "out", out.device)         # dtype
    with pytest.raises(ValueError):
        dg._out(out, (torch.bfloat16,), (4, 3), "out", out.device)        # shape
    with pytest.raises(ValueError):
        dg._out(out.t(), (torch.bfloat16,), (4, 3), "out", out.device)    # not contiguous
    with pytest.raises(ValueError):
        dg._out(out, (torch.bfloat16,), (3, 4), "out", torch.device("meta"))


@pytest.mark.parametrize("env,expect_grid,expect_pdl", [
    ({}, 148, 1),
    ({"DG_NUM_SMS": "64"}, 64, 1),
    ({"DG_TC_UTIL": "50"}, 74, 1),
    ({"DG_TC_UTIL": "abc", "DG_PDL": "0"}, 148, 0),     # malformed value ignored
    ({"DG_TC_UTIL": "0"}, 148, 1),                     # out of range ignored
])
def test_knobs_take_environment_defaults(lib, env, expect_grid, expect_pdl):
    """DG_NUM_SMS / DG_TC_UTIL / DG_PDL set the knobs' initial values when the
    library loads (a fresh process per case; no GPU: 148 SMs assumed)."""
    import os
    import sys

    code = ("from moe_grouped_gemm_05_b200 import binding as dg; lib = dg.load(); "
            "print(dg.describe_config('dense', 4096, 7168, 2048).split('/')[-1], lib.dg_set_pdl(1))")
    clean = {k: v for k, v in os.environ.items() if not k.startswith("DG_")}
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300,
                         env={**clean, **env, "CUDA_VISIBLE_DEVICES": ""},
                         cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    assert out.returncode == 0, out.stderr[-2000:]
    grid, pdl = out.stdout.split()
    assert int(grid) == expect_grid, out.stdout
    assert int(pdl) == expect_pdl


def test_every_other_entry_point_rejects_bad_arguments_on_the_host(lib):
    """Argument errors come back as status codes before any device query or
    launch, for the entry points not covered above (runs without a GPU)."""
    odd4 = P(0x10004)   # 4-byte but not 16-byte aligned
    for name in ("dg_fp8_gemm_nn", "dg_fp8_gemm_tn", "dg_fp8_gemm_tt"):
        f = getattr(lib, name)
        assert f(P(0), GOOD, GOOD, GOOD, GOOD, 128, 256, 256, None) == -1, name
        assert f(GOOD, GOOD, GOOD, GOOD, P(0x10008), 128, 256, 256, None) == -3, name
        assert f(GOOD, GOOD, GOOD, GOOD, GOOD, 128, 256, 100, None) == -2, name
        assert f(GOOD, GOOD, GOOD, GOOD, GOOD, 128, 200, 256, None) == -2, name
        assert f(GOOD, GOOD, GOOD, GOOD, GOOD, -1, 256, 256, None) == -2, name
        assert f(GOOD, GOOD, GOOD, GOOD, GOOD, 0, 256, 256, None) == 0, name
    # A stored [K][M] (TN, TT): its rows are M bytes, which must be a multiple of 16
    assert lib.dg_fp8_gemm_tn(GOOD, GOOD, GOOD, GOOD, GOOD, 120, 256, 256, None) == -2
    assert lib.dg_fp8_gemm_tt(GOOD, GOOD, GOOD, GOOD, GOOD, 120, 256, 256, None) == -2

    ex = lib.dg_fp8_gemm_nt_ex
    assert ex(GOOD, GOOD, GOOD, GOOD, None, GOOD, 128, 256, 256, 64, 0, None) == -4   # granularity 1 or 128
    assert ex(GOOD, GOOD, GOOD, GOOD, None, GOOD, 128, 256, 256, 128, 2, None) == -4  # d_is_fp32 0 or 1
    assert ex(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 128, 256, 256, 128, 0, None) == -4  # C needs an FP32 d
    assert ex(GOOD, GOOD, GOOD, GOOD, P(0x10008), GOOD, 128, 256, 256, 128, 1, None) == -3
    assert ex(GOOD, GOOD, GOOD, GOOD, None, GOOD, 0, 256, 256, 1, 1, None) == 0

    # fp32 A scales need 4-byte alignment only; packed words need 16
    f32 = lib.dg_fp8_gemm_nt_fp32sfa
    assert f32(GOOD, odd4, GOOD, GOOD, GOOD, 0, 256, 256, None) == 0
    assert f32(GOOD, P(0x10002), GOOD, GOOD, GOOD, 0, 256, 256, None) == -3
    assert lib.dg_fp8_gemm_nt(GOOD, odd4, GOOD, GOOD, GOOD, 0, 256, 256, None) == -3
    cf = lib.dg_m_grouped_fp8_gemm_nt_contiguous_fp32sfa
    assert cf(GOOD, odd4, GOOD, GOOD, GOOD, GOOD, 0, 256, 256, 4, None) == 0
    assert cf(GOOD, odd4, GOOD, GOOD, GOOD, GOOD, 200, 256, 256, 4, None) == -2
    mf = lib.dg_m_grouped_fp8_gemm_nt_masked_fp32sfa
    assert mf(GOOD, odd4, GOOD, GOOD, GOOD, P(0), 4, 256, 256, 256, None) == -1
    assert mf(GOOD, odd4, GOOD, GOOD, GOOD, GOOD, 4, 0, 256, 256, None) == 0

    q = lib.dg_quantize_fp8_1x128
    assert q(P(0), 0, GOOD, GOOD, 1, 128, 256, None) == -1
    assert q(GOOD, 2, GOOD, GOOD, 1, 128, 256, None) == -4                 # dtype code 0 (bf16) or 1 (fp32)
    assert q(GOOD, 0, odd4, GOOD, 1, 128, 256, None) == -3
    assert q(GOOD, 0, GOOD, GOOD, 1, 128, 200, None) == -2
    assert q(GOOD, 0, GOOD, GOOD, -1, 128, 256, None) == -2
    assert q(GOOD, 0, GOOD, GOOD, 0, 128, 256, None) == 0                  # empty batch: nothing to do

    cap = lib.dg_moe_permute_capacity
    assert cap(100, 2, 4) == (200 + 127 * 4 + 127) // 128 * 128
    assert cap(-1, 2, 4) == -2 and cap(10, 0, 4) == -2 and cap(10, 2, 0) == -2
    perm = lib.dg_moe_permute
    c = cap(100, 2, 4)
    args = lambda **kw: [kw.get("ids", GOOD), kw.get("T", 100), kw.get("topk", 2), kw.get("G", 4), kw.get("q", GOOD),
                         GOOD, kw.get("K", 256), GOOD, GOOD, GOOD, GOOD, GOOD, kw.get("M_cap", c), None]
    assert perm(*args(ids=P(0))) == -1
    assert perm(*args(q=odd4)) == -3
    assert perm(*args(G=1025)) == -2                                       # at most 1024 experts
    assert perm(*args(K=100)) == -2
    assert perm(*args(M_cap=c - 128)) == -2                                # below the capacity
    assert perm(*args(M_cap=c + 64)) == -2                                 # not a multiple of 128

    comb = lib.dg_moe_unpermute_combine
    assert comb(P(0), GOOD, None, 10, 2, 256, GOOD, None) == -1
    assert comb(GOOD, GOOD, None, 10, 2, 256, odd4, None) == -3
    assert comb(GOOD, GOOD, None, 10, 0, 256, GOOD, None) == -2
    assert comb(GOOD, GOOD, None, 10, 2, 200, GOOD, None) == -2
    assert comb(GOOD, GOOD, None, 0, 2, 256, GOOD, None) == 0              # no tokens: nothing to do


def test_last_error_and_forced_config_are_per_thread(lib):
    """dg_get_last_error() and dg_set_config() are per host thread: one
    thread's failure text and forced tiles do not leak into another's."""
    import threading

    from moe_grouped_gemm_05_b200 import binding as dg

    barrier = threading.Barrier(2)
    seen = {}

    def worker(name, K, force):
        if force:
            assert lib.dg_set_config(128, 1, 1) == 0
        assert _dense(lib, K=K) == -2
        barrier.wait()                    # both threads have failed before either reads its text
        seen[name] = (lib.dg_get_last_error().decode(), dg.describe_config("dense", 4096, 7168, 2048))
        barrier.wait()
        lib.dg_set_config(0, 0, 0)

    threads = [threading.Thread(target=worker, args=("a", 100, True)),
               threading.Thread(target=worker, args=("b", 300, False))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=60)
    assert "K=100" in seen["a"][0] and "K=300" in seen["b"][0]
    assert seen["a"][1].startswith("128x128x6/")                      # forced on thread a only
    assert seen["b"][1] == "256x224x6(2cta)(2pipe)/148"              # thread b keeps the heuristic
