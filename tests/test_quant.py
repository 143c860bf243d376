"""The FP8 (e4m3) weight converter (quant.py, through the library's per-row quantiser): codes and
scales against the e4m3 format's definition and the oracle's quantiser (needs a B200)."""
import numpy as np
import pytest
import torch

from fine_grained_mixture_route_b200 import quant
from fine_grained_mixture_route_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _e4m3_values():
    """All finite e4m3 values from the format's definition: 1 sign, 4 exponent (bias 7) and
    3 mantissa bits, subnormals at exponent 0, no infinities, S.1111.111 is NaN."""
    vals = set()
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            vals.add(v)
            vals.add(-v)
    return torch.tensor(sorted(vals), dtype=torch.float64)


def test_codes_are_nearest_e4m3_values():
    grid = _e4m3_values()
    assert grid.max().item() == quant.E4M3_MAX
    g = torch.Generator().manual_seed(0)
    w = (torch.randn(64, 304, generator=g) * 0.006).bfloat16()
    q, s = quant.quantize_rows(w.cuda())
    q, s = q.cpu(), s.cpu()
    deq = quant.dequantize_rows(q, s).double()
    r = (w.float() / s.unsqueeze(-1)).double()           # the value the quantizer rounds (fp32)
    codes = q.view(torch.float8_e4m3fn).double()
    # every code is an e4m3 value, and the nearest one to w / scale (ties aside)
    idx = torch.searchsorted(grid, codes.reshape(-1).contiguous())
    assert torch.equal(grid[idx.clamp(max=grid.numel() - 1)], codes.reshape(-1))
    dist = (grid.unsqueeze(0) - r.reshape(-1, 1)).abs()
    best = dist.min(dim=1).values
    assert torch.all((codes.reshape(-1) - r.reshape(-1)).abs() <= best + 1e-12)
    # the row maximum maps to +-448 exactly, and the scale is the row maximum / 448
    assert torch.allclose(codes.abs().amax(dim=1), torch.full((64,), 448.0, dtype=torch.float64))
    assert torch.equal(s, w.float().abs().amax(dim=1) / 448.0)
    # relative error of a normal e4m3 value is at most 2^-4
    big = r.abs() >= 2.0 ** -6
    rel = ((deq - w.double()).abs() / w.double().abs())[big]
    assert rel.max().item() <= 2.0 ** -4 + 1e-12


def test_zero_rows_and_stack_round_trip():
    w = torch.zeros(3, 8, 16, dtype=torch.bfloat16)
    w[1] = torch.linspace(-1, 1, 128).reshape(8, 16)
    q, s = quant.quantize_rows(w.cuda())
    assert torch.equal(s[0].cpu(), torch.ones(8))
    assert torch.equal(quant.dequantize_rows(q, s)[0].cpu(), torch.zeros(8, 16))
    cfg = W.scaled(W.CONFIGS["decode"], T=8, d=64, n_experts=4, inter=32, inter_shared=32)
    st = W.make_expert_stack(cfg, False, "cuda")
    qs = quant.quantize_stack(st)
    assert qs["w1"].dtype == torch.uint8 and qs["s2"].shape == (4, 64)
    back = quant.dequantize_stack(qs)
    for k in ("w1", "w3", "w2"):
        err = (back[k] - st[k].float()).abs().max() / st[k].float().abs().max()
        assert err.item() < 2.0 ** -4
    assert back["b1"] is st["b1"]


def test_weight_codes_match_the_oracle_quantiser():
    """The converter and the oracle's per-row quantiser (written separately from the e4m3
    definition) give the same codes and scales."""
    import oracle.moe_oracle as O
    g = torch.Generator().manual_seed(3)
    w = (torch.randn(40, 96, generator=g) * torch.exp2(torch.empty(40, 1).uniform_(-14, 6, generator=g)))
    w[4] = 0.0
    w = w.bfloat16()
    q, s = quant.quantize_rows(w.cuda())
    q_ref, s_ref = O.quantize_rows_e4m3(w.double().numpy())
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(O.e4m3_decode(q.cpu().numpy()), q_ref)


def test_quantized_w1_w3_share_one_buffer():
    cfg = W.scaled(W.CONFIGS["small"], T=8, d=64, n_experts=4, inter=32, inter_shared=32)
    q = quant.quantize_stack(W.make_expert_stack(cfg, False, "cuda"))
    w1, w3 = q["w1"], q["w3"]
    assert w1.dtype == torch.uint8 and w1.is_contiguous() and w3.is_contiguous()
    assert w3.data_ptr() - w1.data_ptr() == w1.numel()
    # the codes are the per-matrix quantisation of each, unchanged by the shared placement
    ref1, _ = quant.quantize_rows(W.make_expert_stack(cfg, False, "cuda")["w1"])
    assert torch.equal(w1, ref1)


def test_converter_needs_bf16_on_the_gpu():
    with pytest.raises(ValueError):
        quant.quantize_rows(torch.zeros(4, 8, dtype=torch.bfloat16))          # host tensor
    with pytest.raises(ValueError):
        quant.quantize_rows(torch.zeros(4, 8, device="cuda"))                  # fp32
