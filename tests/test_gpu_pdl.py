"""Programmatic dependent launch keeps stream order: a chain of dependent
kernels (quantise -> permute -> contiguous grouped GEMM -> combine, and a
scale pack feeding a dense GEMM) gives bit-identical results with the
launch attribute on and off, eagerly and replayed from a CUDA graph with
new inputs copied into the captured buffers."""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import synth

from helpers import bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    prev = dg.set_pdl(True)
    dg.set_config(0)
    dg.get_device_error()
    yield
    dg.set_pdl(prev)


T, TOPK, G, K, N = 512, 2, 6, 1024, 384


def _inputs(seed):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.permutation(G)[:TOPK] for _ in range(T)]).astype(np.int32)
    x = torch.from_numpy(synth.normal(seed, T * K).reshape(T, K)).to(torch.bfloat16)
    gate = rng.random((T, TOPK)).astype(np.float32)
    return torch.from_numpy(ids), x, torch.from_numpy(gate)


def _weights():
    w = synth.contiguous_problem(G, N, K, rows=0, seed=11, counts=[1] * G)
    sb, _ = oracle.pack_sf_ue8m0(w.sfb)
    return torch.from_numpy(w.b).cuda().view(torch.float8_e4m3fn), torch.from_numpy(sb).cuda()


class Chain:
    """The MoE chain on fixed device buffers (so a graph can be captured over it)."""

    def __init__(self):
        self.b, self.sfb = _weights()
        self.ids = torch.empty((T, TOPK), dtype=torch.int32, device="cuda")
        self.x = torch.empty((T, K), dtype=torch.bfloat16, device="cuda")
        self.gate = torch.empty((T, TOPK), dtype=torch.float32, device="cuda")
        self.q = torch.empty((T, K), dtype=torch.float8_e4m3fn, device="cuda")
        self.sfa = torch.empty(dg.packed_sf_words(T, K // 128), dtype=torch.int32, device="cuda")
        cap = dg.load().dg_moe_permute_capacity(T, TOPK, G)
        self.per = {"a": torch.empty((cap, K), dtype=torch.float8_e4m3fn, device="cuda"),
                    "sfa": torch.empty(dg.packed_sf_words(cap, K // 128), dtype=torch.int32, device="cuda"),
                    "m_indices": torch.empty(cap, dtype=torch.int32, device="cuda"),
                    "row_of": torch.empty((T, TOPK), dtype=torch.int32, device="cuda"),
                    "src_of": torch.empty(cap, dtype=torch.int32, device="cuda")}
        self.d = torch.empty((cap, N), dtype=torch.bfloat16, device="cuda")
        self.out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")

    def load(self, ids, x, gate):
        self.ids.copy_(ids)
        self.x.copy_(x)
        self.gate.copy_(gate)

    def run(self):
        dg.quantize_fp8_1x128(self.x, q=self.q, sf=self.sfa)
        dg.moe_permute(self.ids, G, self.q, self.sfa, out=self.per)
        dg.m_grouped_fp8_gemm_nt_contiguous(self.per["a"], self.per["sfa"], self.b, self.sfb,
                                            self.per["m_indices"], self.d)
        dg.moe_unpermute_combine(self.d, self.per["row_of"], self.gate, out=self.out)

    def result(self):
        torch.cuda.synchronize()
        return bits(self.out).copy()


def test_moe_chain_same_bits_with_and_without_pdl():
    chain = Chain()
    chain.load(*_inputs(1))
    dg.set_pdl(False)
    chain.run()
    ref = chain.result()
    dg.set_pdl(True)
    for _ in range(3):
        chain.out.zero_()
        chain.run()
        assert np.array_equal(chain.result(), ref)
    assert dg.get_device_error() == 0


def test_moe_chain_graph_with_pdl_matches_eager():
    chain = Chain()
    refs = []
    dg.set_pdl(False)
    for seed in (2, 3):
        chain.load(*_inputs(seed))
        chain.run()
        refs.append(chain.result())
    dg.set_pdl(True)
    chain.load(*_inputs(2))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        chain.run()  # warm-up outside capture (tensor maps, attributes)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            chain.run()
    for seed, ref in zip((2, 3), refs):
        chain.load(*_inputs(seed))
        chain.out.zero_()
        g.replay()
        assert np.array_equal(chain.result(), ref), f"seed {seed}"
    assert dg.get_device_error() == 0


def test_pack_then_gemm_back_to_back():
    """The packing kernel rewrites the scale words a GEMM just read; with PDL
    the next pack must still wait for that GEMM.  Alternate two scale sets."""
    M, Nd, Kd = 512, 1024, 1024
    p = synth.dense_problem(M, Nd, Kd, seed=12)
    a = torch.from_numpy(p.a).cuda().view(torch.float8_e4m3fn)
    b = torch.from_numpy(p.b).cuda().view(torch.float8_e4m3fn)
    sfb = dg.pack_sf_ue8m0(torch.from_numpy(p.sfb).cuda())
    sf_sets = [torch.from_numpy(p.sfa).cuda(), torch.from_numpy(p.sfa * 2.0).cuda()]
    sfa = torch.empty(dg.packed_sf_words(M, Kd // 128), dtype=torch.int32, device="cuda")
    outs = [torch.empty((M, Nd), dtype=torch.bfloat16, device="cuda") for _ in range(6)]
    for i in range(6):
        dg.pack_sf_ue8m0(sf_sets[i % 2], out=sfa)
        dg.fp8_gemm_nt(a, sfa, b, sfb, outs[i])
    torch.cuda.synchronize()
    base = bits(outs[0])
    doubled = bits(outs[1])
    assert not np.array_equal(base, doubled)
    for i in range(2, 6):
        assert np.array_equal(bits(outs[i]), base if i % 2 == 0 else doubled), f"launch {i}"
