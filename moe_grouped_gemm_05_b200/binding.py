"""Thin ctypes binding of libdg.so (argument marshalling only).

Every step of the GEMM runs in the library's CUDA kernels; this module checks
tensor dtypes/shapes, passes raw device pointers and the current CUDA stream,
and turns negative status codes into exceptions.  Tensors come from PyTorch
(device memory and streams only).  If the library is missing the first call
raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdg.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "dg.h")

DG_OK = 0
DG_ERR_NULL = -1
DG_ERR_SHAPE = -2
DG_ERR_ALIGN = -3
DG_ERR_UNSUPPORTED = -4
DG_ERR_CUDA = -5

DG_DEVERR_BAD_SCALE = 0x1
DG_DEVERR_BAD_EXPERT = 0x2
DG_DEVERR_BAD_MASKED_M = 0x4
DG_DEVERR_MIXED_TILE = 0x8
DG_DEVERR_TIMEOUT = 0x10

_lib = None


class DGError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"dg status {code}: {msg}")
        self.code = code


def load() -> ctypes.CDLL:
    """Loads libdg.so once (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m moe_grouped_gemm_05_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32p, i = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
    lib.dg_fp8_gemm_nt.argtypes = [vp, i32p, vp, i32p, vp, i, i, i, vp]
    lib.dg_fp8_gemm_nt_fp32sfa.argtypes = [vp, vp, vp, i32p, vp, i, i, i, vp]
    lib.dg_m_grouped_fp8_gemm_nt_contiguous_fp32sfa.argtypes = [vp, vp, vp, i32p, vp, i32p, i, i, i, i, vp]
    lib.dg_m_grouped_fp8_gemm_nt_masked_fp32sfa.argtypes = [vp, vp, vp, i32p, vp, i32p, i, i, i, i, vp]
    for name in ("dg_fp8_gemm_nn", "dg_fp8_gemm_tn", "dg_fp8_gemm_tt"):
        getattr(lib, name).argtypes = [vp, i32p, vp, i32p, vp, i, i, i, vp]
    lib.dg_m_grouped_fp8_gemm_nt_contiguous.argtypes = [vp, i32p, vp, i32p, vp, i32p, i, i, i, i, vp]
    lib.dg_m_grouped_fp8_gemm_nt_masked.argtypes = [vp, i32p, vp, i32p, vp, i32p, i, i, i, i, vp]
    lib.dg_pack_sf_ue8m0.argtypes = [vp, i32p, i, i, i, vp]
    lib.dg_quantize_fp8_1x128.argtypes = [vp, i, vp, i32p, i, i, i, vp]
    lib.dg_fp8_gemm_nt_ex.argtypes = [vp, i32p, vp, i32p, vp, vp, i, i, i, i, i, vp]
    lib.dg_moe_permute_capacity.argtypes = [i, i, i]
    lib.dg_moe_permute.argtypes = [i32p, i, i, i, vp, i32p, i, vp, i32p, i32p, i32p, i32p, i, vp]
    lib.dg_moe_unpermute_combine.argtypes = [vp, i32p, vp, i, i, i, vp, vp]
    lib.dg_packed_sf_words.argtypes = [i, i]
    lib.dg_packed_sf_words.restype = ctypes.c_int64
    lib.dg_get_mk_alignment_for_contiguous_layout.argtypes = []
    lib.dg_get_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    lib.dg_set_num_sms.argtypes = [i]
    lib.dg_set_pdl.argtypes = [i]
    lib.dg_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.dg_set_wait_limit_ns.restype = ctypes.c_uint64
    lib.dg_set_tc_util.argtypes = [i]
    lib.dg_get_num_sms.argtypes = []
    lib.dg_set_config.argtypes = [i, i, i]
    lib.dg_describe_config.argtypes = [i, i, i, i, i, ctypes.c_char_p, i]
    lib.dg_get_last_error.restype = ctypes.c_char_p
    for name in ("dg_fp8_gemm_nt", "dg_m_grouped_fp8_gemm_nt_contiguous", "dg_m_grouped_fp8_gemm_nt_masked",
                 "dg_pack_sf_ue8m0", "dg_get_device_error", "dg_set_config", "dg_describe_config",
                 "dg_quantize_fp8_1x128", "dg_fp8_gemm_nt_ex", "dg_moe_permute_capacity", "dg_moe_permute",
                 "dg_moe_unpermute_combine"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def header_functions() -> list[str]:
    """Names of the functions declared in include/dg.h."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_\w+)\s*\(", text)))


def _check(code: int):
    if code != 0:
        raise DGError(code, load().dg_get_last_error().decode())


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _fp8(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise TypeError(f"{name} must be float8_e4m3fn (or its uint8 bytes), got {t.dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return t


def _i32(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous int32 CUDA tensor")
    return t


def packed_sf_words(mn: int, kb: int) -> tuple[int, int]:
    """(rows, cols) of a packed scale matrix: (ceil(kb/4), align4(mn))."""
    return (kb + 3) // 4, (mn + 3) // 4 * 4


def _packed_numel(t, batch: int, mn: int, kb: int, name: str):
    """Packed scale words may come as [kp, mn4] or [batch, kp, mn4]: what the
    kernels read is batch * kp * mn4 words, so the element count must match."""
    kp, mn4 = packed_sf_words(mn, kb)
    if t.numel() != batch * kp * mn4:
        raise ValueError(f"{name} holds {t.numel()} words; expected {batch} x {kp} x {mn4} "
                         f"(batch x ceil(Kb/4) x align4(MN))")


def _same_device(ref, *tensors):
    """All operands of a call live on one device (None entries are skipped)."""
    dev = ref.get_device()
    for t in tensors:
        if t is not None and t.get_device() != dev:
            raise ValueError(f"operands on different devices: {ref.device} and {t.device}")


def _out(t, dtypes, shape, name: str, device):
    """Checks a caller-provided output tensor."""
    if t.dtype not in dtypes or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or t.device != device:
        raise ValueError(f"{name} must be a contiguous {'/'.join(str(d) for d in dtypes)} tensor of shape "
                         f"{tuple(shape)} on {device}")


def pack_sf_ue8m0(sf: torch.Tensor, out=None) -> torch.Tensor:
    """fp32 power-of-two scales [batch?, mn, kb] -> int32 [batch?, ceil(kb/4), align4(mn)] (into `out` if given)."""
    if sf.dtype != torch.float32 or not sf.is_cuda or not sf.is_contiguous():
        raise TypeError("sf must be a contiguous float32 CUDA tensor")
    squeeze = sf.dim() == 2
    s3 = sf.unsqueeze(0) if squeeze else sf
    if s3.dim() != 3:
        raise ValueError("sf must be [mn, kb] or [batch, mn, kb]")
    batch, mn, kb = s3.shape
    kp, mn4 = packed_sf_words(mn, kb)
    if out is None:
        out = torch.empty((batch, kp, mn4), dtype=torch.int32, device=sf.device)
    elif (out.dtype != torch.int32 or not out.is_contiguous() or out.numel() != batch * kp * mn4
          or out.device != sf.device):
        raise ValueError("out must be a contiguous int32 tensor of the packed shape on sf's device")
    _check(load().dg_pack_sf_ue8m0(_ptr(s3), _ptr(out), batch, mn, kb, _stream()))
    if out.dim() == 3 and squeeze:
        return out[0]
    return out


def quantize_fp8_1x128(x: torch.Tensor, q=None, sf=None):
    """Per-token 1x128 FP8 quantisation of x[..., M, K] (bf16 or fp32).

    Returns (q float8_e4m3fn [..., M, K], sf int32 [..., ceil(K/512), align4(M)]),
    the `a` / `sfa` operands of the GEMM entry points.
    """
    if x.dtype not in (torch.bfloat16, torch.float32) or not x.is_cuda or not x.is_contiguous():
        raise TypeError("x must be a contiguous bf16 or fp32 CUDA tensor")
    if x.dim() < 2:
        raise ValueError("x must be [..., M, K]")
    *lead, M, K = x.shape
    batch = 1
    for n in lead:
        batch *= n
    kp, mn4 = packed_sf_words(M, K // 128)
    if q is None:
        q = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    if sf is None:
        sf = torch.empty((*lead, kp, mn4), dtype=torch.int32, device=x.device)
    _out(q, (torch.float8_e4m3fn, torch.uint8), x.shape, "q", x.device)
    _out(sf, (torch.int32,), (*lead, kp, mn4), "sf", x.device)
    _check(load().dg_quantize_fp8_1x128(_ptr(x), 0 if x.dtype == torch.bfloat16 else 1, _ptr(q), _ptr(sf), batch,
                                        M, K, _stream()))
    return q, sf


def _sfa_kind(sfa: torch.Tensor, rows_shape: tuple, K: int) -> bool:
    """True when sfa holds fp32 scales [..rows.., K/128] (packed in the kernel), False for packed int32 words."""
    if sfa.dtype == torch.float32:
        if not sfa.is_cuda or not sfa.is_contiguous() or tuple(sfa.shape) != (*rows_shape, K // 128):
            raise ValueError(f"fp32 sfa must be a contiguous CUDA tensor of shape {(*rows_shape, K // 128)}")
        return True
    _i32(sfa, "sfa")
    return False


def fp8_gemm_nt(a, sfa, b, sfb, d=None) -> torch.Tensor:
    """D[M,N] (bf16) = A[M,K] . B[N,K]^T with 1x128 / 128x128 UE8M0 scales.

    sfa: packed int32 words [ceil(Kb/4), align4(M)], or the fp32 power-of-two scales [M, Kb]
    (then the GEMM packs them itself: no separate packing launch).
    """
    _fp8(a, "a"), _fp8(b, "b"), _i32(sfb, "sfb")
    M, K = a.shape
    N, Kb_ = b.shape
    if Kb_ != K:
        raise ValueError("a and b disagree on K")
    fp32_sfa = _sfa_kind(sfa, (M,), K)
    if (not fp32_sfa and tuple(sfa.shape) != packed_sf_words(M, K // 128)) or \
            tuple(sfb.shape) != packed_sf_words(-(-N // 128), K // 128):
        raise ValueError("packed scale shapes do not match [ceil(Kb/4), align4(MN)]")
    _same_device(a, sfa, b, sfb, d)
    if d is None:
        d = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    elif d.dtype != torch.bfloat16 or tuple(d.shape) != (M, N) or not d.is_contiguous():
        raise ValueError("d must be a contiguous bf16 [M, N] tensor")
    fn = load().dg_fp8_gemm_nt_fp32sfa if fp32_sfa else load().dg_fp8_gemm_nt
    _check(fn(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), M, N, K, _stream()))
    return d


def fp8_gemm(layout: str, a, sfa, b, sfb, d=None) -> torch.Tensor:
    """D[M,N] (bf16) = A . B^T with the operands stored in `layout` ("nt", "nn", "tn" or "tt").

    First letter LHS, second RHS, N = not transposed, T = transposed:
    a is A [M,K] for "n?" and A^T [K,M] for "t?"; b is B [N,K] for "?t" and B^T [K,N] for "?n".
    """
    if layout not in ("nt", "nn", "tn", "tt"):
        raise ValueError(f"unknown layout {layout!r}")
    _fp8(a, "a"), _fp8(b, "b"), _i32(sfa, "sfa"), _i32(sfb, "sfb")
    if not (a.is_contiguous() and b.is_contiguous()):
        raise ValueError("a and b must be contiguous")
    K, M = a.shape if layout[0] == "t" else a.shape[::-1]
    K2, N = b.shape if layout[1] == "n" else b.shape[::-1]
    if K2 != K:
        raise ValueError("a and b disagree on K")
    if tuple(sfa.shape) != packed_sf_words(M, K // 128) or tuple(sfb.shape) != packed_sf_words(-(-N // 128), K // 128):
        raise ValueError("packed scale shapes do not match [ceil(Kb/4), align4(MN)]")
    _same_device(a, sfa, b, sfb, d)
    if d is None:
        d = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    elif d.dtype != torch.bfloat16 or tuple(d.shape) != (M, N) or not d.is_contiguous():
        raise ValueError("d must be a contiguous bf16 [M, N] tensor")
    fn = getattr(load(), f"dg_fp8_gemm_{layout}")
    _check(fn(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), M, N, K, _stream()))
    return d


def fp8_gemm_nt_ex(a, sfa, b, sfb, c=None, d=None, recipe_b: int = 128, out_dtype=torch.bfloat16) -> torch.Tensor:
    """D = A . B^T (+ C).  recipe_b: rows of B per scale (128 = 128x128 blocks, 1 = per-row "1D1D").

    out_dtype bf16 or float32; c (float32 [M, N]) requires a float32 output.
    """
    _fp8(a, "a"), _fp8(b, "b"), _i32(sfa, "sfa"), _i32(sfb, "sfb")
    M, K = a.shape
    N, Kb_ = b.shape
    if Kb_ != K:
        raise ValueError("a and b disagree on K")
    if tuple(sfb.shape) != packed_sf_words(-(-N // recipe_b), K // 128) or tuple(sfa.shape) != packed_sf_words(M, K // 128):
        raise ValueError("packed scale shapes do not match the recipe")
    if c is not None and (c.dtype != torch.float32 or tuple(c.shape) != (M, N) or not c.is_contiguous()):
        raise ValueError("c must be a contiguous float32 [M, N] tensor")
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    _same_device(a, sfa, b, sfb, c, d)
    if d is None:
        d = torch.empty((M, N), dtype=out_dtype, device=a.device)
    else:
        _out(d, (torch.bfloat16, torch.float32), (M, N), "d", a.device)
    _check(load().dg_fp8_gemm_nt_ex(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(c) if c is not None else None,
                                    _ptr(d), M, N, K, recipe_b, 1 if d.dtype == torch.float32 else 0, _stream()))
    return d


def m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, m_indices, d=None) -> torch.Tensor:
    """Contiguous-layout grouped GEMM: D[m] = A[m] . B[m_indices[m]]^T; -1 rows untouched.

    sfa: packed words or fp32 scales [M_total, Kb] (packed in the kernel)."""
    _fp8(a, "a"), _fp8(b, "b"), _i32(sfb, "sfb"), _i32(m_indices, "m_indices")
    M, K = a.shape
    G, N, Kb_ = b.shape
    if Kb_ != K or m_indices.shape != (M,):
        raise ValueError("shape mismatch")
    fp32_sfa = _sfa_kind(sfa, (M,), K)
    if not fp32_sfa:
        _packed_numel(sfa, 1, M, K // 128, "sfa")
    _packed_numel(sfb, G, -(-N // 128), K // 128, "sfb")
    _same_device(a, sfa, b, sfb, m_indices, d)
    if d is None:
        d = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    elif d.dtype != torch.bfloat16 or tuple(d.shape) != (M, N) or not d.is_contiguous():
        raise ValueError("d must be a contiguous bf16 [M_total, N] tensor")
    fn = load().dg_m_grouped_fp8_gemm_nt_contiguous_fp32sfa if fp32_sfa else load().dg_m_grouped_fp8_gemm_nt_contiguous
    _check(fn(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), _ptr(m_indices), M, N, K, G, _stream()))
    return d


def m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, masked_m, d=None) -> torch.Tensor:
    """Masked-layout grouped GEMM: rows m < masked_m[g] of expert g; other rows untouched.

    sfa: packed words or fp32 scales [G, M_max, Kb] (packed in the kernel)."""
    _fp8(a, "a"), _fp8(b, "b"), _i32(sfb, "sfb"), _i32(masked_m, "masked_m")
    G, M_max, K = a.shape
    Gb, N, Kb_ = b.shape
    if Gb != G or Kb_ != K or masked_m.shape != (G,):
        raise ValueError("shape mismatch")
    fp32_sfa = _sfa_kind(sfa, (G, M_max), K)
    if not fp32_sfa:
        _packed_numel(sfa, G, M_max, K // 128, "sfa")
    _packed_numel(sfb, G, -(-N // 128), K // 128, "sfb")
    _same_device(a, sfa, b, sfb, masked_m, d)
    if d is None:
        d = torch.empty((G, M_max, N), dtype=torch.bfloat16, device=a.device)
    elif d.dtype != torch.bfloat16 or tuple(d.shape) != (G, M_max, N) or not d.is_contiguous():
        raise ValueError("d must be a contiguous bf16 [G, M_max, N] tensor")
    fn = load().dg_m_grouped_fp8_gemm_nt_masked_fp32sfa if fp32_sfa else load().dg_m_grouped_fp8_gemm_nt_masked
    _check(fn(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(d), _ptr(masked_m), G, M_max, N, K, _stream()))
    return d


def moe_permute(topk_ids: torch.Tensor, num_experts: int, q: torch.Tensor, sfa: torch.Tensor, out=None):
    """Contiguous-layout permutation of routed tokens.

    Returns a dict with a (float8 [M_cap, K]), sfa (int32 [kp, M_cap]), m_indices, src_of ([M_cap]) and
    row_of ([T, topk]); a / sfa / m_indices are the operands of m_grouped_fp8_gemm_nt_contiguous.
    `out`, if given, is such a dict of preallocated tensors (M_cap = dg_moe_permute_capacity).
    """
    _i32(topk_ids, "topk_ids"), _fp8(q, "q"), _i32(sfa, "sfa")
    T, topk = topk_ids.shape
    if q.dim() != 2 or q.shape[0] != T:
        raise ValueError(f"q must be [T, K] with T = {T} rows, one per token of topk_ids")
    K = q.shape[1]
    _packed_numel(sfa, 1, T, K // 128, "sfa")
    _same_device(q, topk_ids, sfa)
    cap = load().dg_moe_permute_capacity(T, topk, num_experts)
    if cap < 0:
        _check(cap)
    kp = (K // 128 + 3) // 4
    dev = q.device
    if out is None:
        out = {
            "a": torch.empty((cap, K), dtype=torch.float8_e4m3fn, device=dev),
            "sfa": torch.empty((kp, cap), dtype=torch.int32, device=dev),
            "m_indices": torch.empty((cap,), dtype=torch.int32, device=dev),
            "src_of": torch.empty((cap,), dtype=torch.int32, device=dev),
            "row_of": torch.empty((T, topk), dtype=torch.int32, device=dev),
        }
    else:
        want = {"a": ((torch.float8_e4m3fn, torch.uint8), (cap, K)), "sfa": ((torch.int32,), (kp, cap)),
                "m_indices": ((torch.int32,), (cap,)), "src_of": ((torch.int32,), (cap,)),
                "row_of": ((torch.int32,), (T, topk))}
        for key, (dtypes, shape) in want.items():
            if key not in out:
                raise ValueError(f"out[{key!r}] is missing")
            _out(out[key], dtypes, shape, f"out[{key!r}]", dev)
    _check(load().dg_moe_permute(_ptr(topk_ids), T, topk, num_experts, _ptr(q), _ptr(sfa), K, _ptr(out["a"]),
                                 _ptr(out["sfa"]), _ptr(out["m_indices"]), _ptr(out["row_of"]), _ptr(out["src_of"]),
                                 cap, _stream()))
    return out


def moe_unpermute_combine(d_perm: torch.Tensor, row_of: torch.Tensor, weights=None, out=None) -> torch.Tensor:
    """out[t] = sum_s weights[t, s] * d_perm[row_of[t, s]] (bf16, FP32 sums)."""
    if d_perm.dtype != torch.bfloat16 or not d_perm.is_contiguous() or not d_perm.is_cuda or d_perm.dim() != 2:
        raise TypeError("d_perm must be a contiguous bf16 [rows, N] CUDA tensor")
    _i32(row_of, "row_of")
    T, topk = row_of.shape
    N = d_perm.shape[1]
    if weights is not None:
        _out(weights, (torch.float32,), (T, topk), "weights", d_perm.device)
    _same_device(d_perm, row_of)
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=d_perm.device)
    else:
        _out(out, (torch.bfloat16,), (T, N), "out", d_perm.device)
    _check(load().dg_moe_unpermute_combine(_ptr(d_perm), _ptr(row_of), _ptr(weights) if weights is not None else None,
                                           T, topk, N, _ptr(out), _stream()))
    return out


def get_device_error() -> int:
    """Returns and clears the device error word (atomically, after the current stream's work)."""
    v = ctypes.c_int(0)
    _check(load().dg_get_device_error(_stream(), ctypes.byref(v)))
    return v.value


def set_wait_limit_ns(ns: int) -> int:
    """Sets the time limit of each pipeline wait in the GEMM kernels; returns the previous one."""
    if ns < 0:
        raise ValueError("the wait limit is a non-negative number of nanoseconds")
    return int(load().dg_set_wait_limit_ns(ns))


def set_num_sms(n: int) -> int:
    return load().dg_set_num_sms(n)


def set_tc_util(percent: int) -> int:
    """Caps the share of the GPU's SMs (tensor cores) a call may occupy; returns the previous percent."""
    prev = load().dg_set_tc_util(percent)
    if prev < 0:
        _check(prev)
    return prev


def set_pdl(enable: bool) -> bool:
    """Programmatic dependent launch on/off for the library's kernels; returns the previous setting."""
    return bool(load().dg_set_pdl(1 if enable else 0))


def set_config(block_n: int, ctas: int = 0, pipes: int = 0) -> None:
    """Forces the N tile width, 1- or 2-CTA tiles and 1 or 2 pipelines per CTA (block_n=0: heuristic)."""
    _check(load().dg_set_config(block_n, ctas, pipes))


def describe_config(kind: str, M: int, N: int, K: int, num_groups: int = 1) -> str:
    buf = ctypes.create_string_buffer(64)
    k = {"dense": 0, "contiguous": 1, "masked": 2}[kind]
    _check(load().dg_describe_config(k, M, N, K, num_groups, buf, 64))
    return buf.value.decode()


def get_mk_alignment_for_contiguous_layout() -> int:
    return load().dg_get_mk_alignment_for_contiguous_layout()
