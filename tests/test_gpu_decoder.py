"""Synthetic decoder forward (24 layers x 12 W4A4 GEMM calls): every
recorded call is checked against the oracle on the GPU's own inputs
(teacher forcing) -- two layers at M = 1 and 16, all 288 calls of the full
24-layer forward at M = 1, sampled rows at M = 256 -- and the CUDA-graph
replay must reproduce the eager forward bit for bit."""
import numpy as np
import pytest
import torch

from tests.parity import gemm_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dec():
    from mxfp4_block_scaled_fp4_b200.decoder import SyntheticDecoder
    return SyntheticDecoder("cuda", layers=2)


def _check_calls(orc, dec, record, rows=None):
    for li, name, x, y in record:
        w = dec.wb[li][name]
        xs = x if rows is None else x[rows]
        ca, sa, ga = orc.quantize(x.cpu(), 0)               # global scale of the whole input
        if rows is not None:
            ca, sa, ga = orc.quantize(xs.cpu(), 0, ga)
        cw, sw, gw = orc.quantize(w.cpu(), 0)
        c_ref = orc.gemm(orc.dequant(ca, sa, 0, ga), orc.dequant(cw, sw, 0, gw))
        yy = y if rows is None else y[rows]
        ok, worst, where = gemm_close(yy, c_ref, torch.bfloat16)
        assert ok, f"layer {li} {name}: worst err/bound {worst:.3g} at {where}"


@pytest.mark.parametrize("M", [1, 16])
def test_every_call_teacher_forced(orc, dec, M):
    x = torch.randn(M, 2880, generator=torch.Generator().manual_seed(M)).to(torch.bfloat16).cuda()
    dec.record = []
    dec.forward_fp4(x)
    torch.cuda.synchronize()
    rec, dec.record = dec.record, None
    assert len(rec) == 2 * 12
    _check_calls(orc, dec, rec)


def test_large_m_calls_sampled_rows(orc, dec):
    M = 256
    x = torch.randn(M, 2880, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16).cuda()
    dec.record = []
    dec.forward_fp4(x)
    torch.cuda.synchronize()
    rec, dec.record = dec.record, None
    rows = torch.tensor(np.random.default_rng(0).choice(M, 32, replace=False))
    _check_calls(orc, dec, [rec[i] for i in (0, 3, 5, 11, 12, 23)], rows=rows)


def test_graph_replay_equals_eager(dec):
    x = torch.randn(16, 2880, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    eager = dec.forward_fp4(x.clone())
    xs = x.clone()
    g, out = dec.capture(dec.forward_fp4, xs)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    assert torch.isfinite(out.float()).all()


def test_full_depth_every_call_teacher_forced(orc):
    """The whole workload's depth: 24 layers, all 288 calls of an M=1
    forward checked against the oracle on their recorded inputs."""
    from mxfp4_block_scaled_fp4_b200.decoder import SyntheticDecoder
    dec24 = SyntheticDecoder("cuda")
    assert dec24.layers == 24
    x = torch.randn(1, 2880, generator=torch.Generator().manual_seed(11)).to(torch.bfloat16).cuda()
    dec24.record = []
    out = dec24.forward_fp4(x)
    torch.cuda.synchronize()
    rec, dec24.record = dec24.record, None
    assert len(rec) == 288
    assert torch.isfinite(out.float()).all()
    _check_calls(orc, dec24, rec)
