"""GPU parity of the MoE permutation (bit exact: deterministic layout, copied
codes and scale words) and the combine, and the whole chain
quantise -> permute -> contiguous grouped GEMM -> combine against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import synth

from helpers import bits, check_close

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dg.get_device_error()


def _routing(T, topk, G, seed, drop=0.1):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.permutation(G)[:topk] for _ in range(T)]).astype(np.int32)
    ids[rng.random((T, topk)) < drop] = -1
    return ids


@pytest.mark.parametrize("T,topk,G,K", [(300, 2, 6, 512), (1, 1, 3, 128), (2048, 8, 32, 640), (64, 4, 256, 256)])
def test_permute_bit_exact(T, topk, G, K):
    ids = _routing(T, topk, G, seed=T + G)
    x = torch.from_numpy(synth.normal(T, T * K).reshape(T, K)).to(torch.bfloat16).cuda()
    q, sfa = dg.quantize_fp8_1x128(x)
    out = dg.moe_permute(torch.from_numpy(ids).cuda(), G, q, sfa)
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0
    m, row_of, src, Mt, bad = oracle.fp8_gemm.moe_permute(ids, G)
    cap = out["m_indices"].shape[0]
    assert cap == oracle.fp8_gemm.moe_permute_capacity(T, topk, G)
    gm = out["m_indices"].cpu().numpy()
    gs = out["src_of"].cpu().numpy()
    assert np.array_equal(gm[:Mt], m) and (gm[Mt:] == -1).all()
    assert np.array_equal(gs[:Mt], src) and (gs[Mt:] == -1).all()
    assert np.array_equal(out["row_of"].cpu().numpy(), row_of)
    valid = np.nonzero(m >= 0)[0]
    qn = q.view(torch.uint8).cpu().numpy()
    an = out["a"].view(torch.uint8).cpu().numpy()
    assert np.array_equal(an[valid], qn[src[valid]])
    sf_src = sfa.cpu().numpy()
    sf_out = out["sfa"].cpu().numpy()
    assert np.array_equal(sf_out[:, valid], sf_src[:, src[valid]])
    assert (sf_out[:, gm < 0] == 0).all()


@pytest.mark.parametrize("T,topk,G,K,zipf", [(20000, 8, 1024, 128, False), (40000, 2, 8, 128, True),
                                               (3000, 4, 63, 256, False), (3000, 4, 64, 256, False)])
def test_permute_many_slots_and_expert_counts(T, topk, G, K, zipf):
    """Routing beyond 65536 slots (each warp of the routing cluster then loads
    its ids in several batches), the largest expert count (1024: the 128 KB
    per-warp count table), and 63 / 64 experts, on either side of the switch
    from match.any to per-bit ballots (6- and 7-bit expert keys)."""
    if zipf:
        ids, _ = synth.topk_routing(T + G, T, topk, G)
    else:
        ids = _routing(T, topk, G, seed=T + G, drop=0.05)
    x = torch.from_numpy(synth.normal(T + 1, T * K).reshape(T, K)).to(torch.bfloat16).cuda()
    q, sfa = dg.quantize_fp8_1x128(x)
    out = dg.moe_permute(torch.from_numpy(ids).cuda(), G, q, sfa)
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0
    m, row_of, src, Mt, bad = oracle.fp8_gemm.moe_permute(ids, G)
    gm, gs = out["m_indices"].cpu().numpy(), out["src_of"].cpu().numpy()
    assert np.array_equal(gm[:Mt], m) and (gm[Mt:] == -1).all()
    assert np.array_equal(gs[:Mt], src) and (gs[Mt:] == -1).all()
    assert np.array_equal(out["row_of"].cpu().numpy(), row_of)
    valid = np.nonzero(m >= 0)[0]
    an = out["a"].view(torch.uint8).cpu().numpy()
    assert np.array_equal(an[valid], q.view(torch.uint8).cpu().numpy()[src[valid]])
    sf_out = out["sfa"].cpu().numpy()
    assert np.array_equal(sf_out[:, valid], sfa.cpu().numpy()[:, src[valid]])
    assert (sf_out[:, gm < 0] == 0).all()


def test_permute_into_prefilled_buffers_over_many_chunks():
    """15000 routed slots (several 4096-slot compaction chunks and a ragged
    last one) with Zipf-weighted top-3 routing, into output buffers filled with
    garbage first: every index, row and scale word the contract defines is
    written, padding and tail scale words included."""
    T, topk, G, K = 5000, 3, 8, 384
    ids, _ = synth.topk_routing(41, T, topk, G)
    ids[::7, 1] = -1  # some unrouted slots
    x = torch.from_numpy(synth.normal(42, T * K).reshape(T, K)).to(torch.bfloat16).cuda()
    q, sfa = dg.quantize_fp8_1x128(x)
    cap = dg.load().dg_moe_permute_capacity(T, topk, G)
    kp = (K // 128 + 3) // 4
    out = {"a": torch.full((cap, K), 0x7E, dtype=torch.uint8, device="cuda").view(torch.float8_e4m3fn),
           "sfa": torch.full((kp, cap), 0x5A5A5A5A, dtype=torch.int32, device="cuda"),
           "m_indices": torch.full((cap,), 77, dtype=torch.int32, device="cuda"),
           "src_of": torch.full((cap,), 77, dtype=torch.int32, device="cuda"),
           "row_of": torch.full((T, topk), 77, dtype=torch.int32, device="cuda")}
    dg.moe_permute(torch.from_numpy(ids).cuda(), G, q, sfa, out=out)
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0
    m, row_of, src, Mt, bad = oracle.fp8_gemm.moe_permute(ids, G)
    gm, gs = out["m_indices"].cpu().numpy(), out["src_of"].cpu().numpy()
    assert np.array_equal(gm[:Mt], m) and (gm[Mt:] == -1).all()
    assert np.array_equal(gs[:Mt], src) and (gs[Mt:] == -1).all()
    assert np.array_equal(out["row_of"].cpu().numpy(), row_of)
    valid = np.nonzero(m >= 0)[0]
    an = out["a"].view(torch.uint8).cpu().numpy()
    assert np.array_equal(an[valid], q.view(torch.uint8).cpu().numpy()[src[valid]])
    sf_out = out["sfa"].cpu().numpy()
    assert np.array_equal(sf_out[:, valid], sfa.cpu().numpy()[:, src[valid]])
    assert (sf_out[:, gm < 0] == 0).all()


def test_permute_no_tokens_marks_every_row_padding():
    K, G, topk = 256, 4, 2
    cap = dg.load().dg_moe_permute_capacity(0, topk, G)
    kp = (K // 128 + 3) // 4
    out = {"a": torch.zeros((cap, K), dtype=torch.float8_e4m3fn, device="cuda"),
           "sfa": torch.full((kp, cap), 9, dtype=torch.int32, device="cuda"),
           "m_indices": torch.full((cap,), 9, dtype=torch.int32, device="cuda"),
           "src_of": torch.full((cap,), 9, dtype=torch.int32, device="cuda"),
           "row_of": torch.zeros((0, topk), dtype=torch.int32, device="cuda")}
    q = torch.zeros((0, K), dtype=torch.float8_e4m3fn, device="cuda")
    sfa = torch.zeros(dg.packed_sf_words(0, K // 128), dtype=torch.int32, device="cuda")
    dg.moe_permute(torch.zeros((0, topk), dtype=torch.int32, device="cuda"), G, q, sfa, out=out)
    torch.cuda.synchronize()
    assert (out["m_indices"].cpu().numpy() == -1).all() and (out["src_of"].cpu().numpy() == -1).all()
    assert (out["sfa"].cpu().numpy() == 0).all()
    assert dg.get_device_error() == 0


def test_permute_flags_bad_ids():
    ids = np.array([[0, 5], [1, -3]], np.int32)
    x = torch.ones((2, 128), dtype=torch.bfloat16, device="cuda")
    q, sfa = dg.quantize_fp8_1x128(x)
    out = dg.moe_permute(torch.from_numpy(ids).cuda(), 2, q, sfa)
    assert dg.get_device_error() & dg.DG_DEVERR_BAD_EXPERT
    assert out["row_of"].cpu().numpy().tolist() == [[0, -1], [128, -1]]


@pytest.mark.parametrize("T,topk,N,weighted", [(1, 1, 16, True), (333, 2, 272, True), (257, 3, 4096, False),
                                                (100, 6, 512, True), (64, 8, 128, True), (50, 9, 96, True),
                                                (20, 12, 48, False)])
def test_combine_matches_oracle(T, topk, N, weighted):
    """The weighted combine on its own, over both slot-pass widths (one slot at
    a time for top-k 1, 2, 3; eight for 6 and 8, and two passes of eight for 9
    and 12), with unrouted slots, a token with no routed slot, and rows of the
    permuted output that no slot reads."""
    rng = np.random.default_rng(T * 31 + topk)
    R = T * topk + 37
    d = torch.from_numpy(synth.normal(T + topk, R * N).reshape(R, N)).to(torch.bfloat16).cuda()
    row_of = rng.permutation(R)[: T * topk].reshape(T, topk).astype(np.int32)
    row_of[rng.random((T, topk)) < 0.15] = -1
    row_of[T // 2] = -1
    gate = rng.random((T, topk)).astype(np.float32) if weighted else None
    out = torch.full((T, N), 7.0, dtype=torch.bfloat16, device="cuda")
    dg.moe_unpermute_combine(d, torch.from_numpy(row_of).cuda(), torch.from_numpy(gate).cuda() if weighted else None,
                             out=out)
    torch.cuda.synchronize()
    ref = oracle.fp8_gemm.moe_unpermute_combine(bits(d), row_of, gate)
    check_close(bits(out), ref, "combine")
    assert (bits(out)[T // 2] == 0).all()


def test_moe_chain_matches_oracle():
    T, topk, G, K, N = 700, 2, 5, 1024, 384
    ids = _routing(T, topk, G, seed=3, drop=0.05)
    x = torch.from_numpy(synth.normal(5, T * K).reshape(T, K)).to(torch.bfloat16)
    w = synth.contiguous_problem(G, N, K, rows=0, seed=6, counts=[1] * G)   # expert weights B[G][N][K]
    sb, _ = oracle.pack_sf_ue8m0(w.sfb)
    gate = np.random.default_rng(7).random((T, topk)).astype(np.float32)
    # GPU chain
    q, sfa = dg.quantize_fp8_1x128(x.cuda())
    per = dg.moe_permute(torch.from_numpy(ids).cuda(), G, q, sfa)
    d = dg.m_grouped_fp8_gemm_nt_contiguous(per["a"], per["sfa"], torch.from_numpy(w.b).cuda().view(torch.float8_e4m3fn),
                                            torch.from_numpy(sb).cuda(), per["m_indices"])
    out = dg.moe_unpermute_combine(d, per["row_of"], torch.from_numpy(gate).cuda())
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0
    # oracle chain
    codes, words = oracle.fp8_gemm.quantize_fp8_1x128(x.float().numpy().astype(np.float64))
    m, row_of, src, Mt, _ = oracle.fp8_gemm.moe_permute(ids, G)
    rows = np.nonzero(m >= 0)[0]
    a_perm = np.zeros((Mt, K), np.uint8)
    a_perm[rows] = codes[src[rows]]
    sa_src = oracle.unpack_sf_ue8m0(words, T, K // 128)[0]
    sa_perm = np.ones((Mt, K // 128), np.float32)
    sa_perm[rows] = np.ldexp(1.0, sa_src[src[rows]].astype(np.int64) - 127)
    sa_words, _ = oracle.pack_sf_ue8m0(sa_perm[None])
    d_ref = np.zeros((Mt, N), np.uint16)
    oracle.m_grouped_fp8_gemm_nt_contiguous(a_perm, sa_words[0], w.b, sb, m, d_ref, G, N, K)
    check_close(bits(d)[rows], d_ref[rows], "permuted grouped GEMM")
    ref = oracle.fp8_gemm.moe_unpermute_combine(d_ref, row_of, gate)
    check_close(bits(out), ref, "combine")
