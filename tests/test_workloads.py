"""The seeded input generator: shapes, determinism and the stated distributions (CPU)."""
import math

import torch

from fine_grained_mixture_route_b200 import workloads as W


def test_configs_match_stated_shapes():
    c = W.CONFIGS
    assert (c["tiny"].T, c["tiny"].d, c["tiny"].n_experts, c["tiny"].inter, c["tiny"].top_k) == (128, 256, 16, 64, 4)
    assert c["tiny"].dtype == torch.float32 and c["tiny"].has_bias
    assert (c["small"].T, c["small"].d, c["small"].n_experts, c["small"].inter, c["small"].top_k) == (2048, 1280, 64, 320, 7)
    assert (c["mid"].n_shared, c["mid"].has_bias, c["mid"].inter) == (2, False, 1408)
    assert (c["decode"].T, c["decode"].d, c["decode"].n_experts, c["decode"].inter, c["decode"].top_k) == (256, 7168, 256, 2048, 8)
    assert c["prefill"].T == 16384 and c["prefill"].centroid_init == "zipf_norm"
    # algorithmic FLOPs of the two V3-shaped layers (router + 3 contractions per pick and shared)
    assert abs(c["prefill"].flops() / 1e12 - 13.05) < 0.01
    assert abs(c["decode"].flops() / 1e12 - 0.204) < 0.001


def test_deterministic_and_slice_regeneration():
    cfg = W.scaled(W.CONFIGS["small"], T=16, d=64, n_experts=8, inter=32, inter_shared=32)
    a = W.make_layer(cfg)
    b = W.make_layer(cfg)
    assert torch.equal(a["x"], b["x"]) and torch.equal(a["centroids"], b["centroids"])
    for k in ("w1", "b1", "w3", "b3", "w2", "b2"):
        assert torch.equal(a["routed"][k], b["routed"][k])
    part = W.make_expert_stack(cfg, False, experts=range(3, 6))
    assert torch.equal(part["w2"], a["routed"]["w2"][3:6])
    assert not torch.equal(a["routed"]["w1"][0], a["routed"]["w1"][1])
    assert not torch.equal(a["routed"]["w1"][0], a["shared"]["w1"][0])
    assert W.make_layer(cfg, seed=1)["x"].ne(a["x"]).any()


def test_distributions():
    cfg = W.scaled(W.CONFIGS["decode"], T=64, d=512, n_experts=32, inter=64, inter_shared=64)
    L = W.make_layer(cfg)
    assert abs(L["x"].float().std().item() - 1.0) < 0.05
    assert abs(L["routed"]["w1"].float().std().item() - 0.006) < 0.0005
    assert abs(L["centroids"].float().std().item() - 0.006) < 0.0005
    mid = W.scaled(W.CONFIGS["mid"], T=8, d=1024, n_experts=64, inter=64, inter_shared=64)
    c = W.make_centroids(mid).float()
    a = math.sqrt(3.0 / 1024)
    assert c.abs().max().item() <= a * 1.01 and abs(c.std().item() - 1 / 32) < 0.002
    assert W.make_expert_stack(mid, False)["b1"] is None


def test_zipf_centroid_norms():
    cfg = W.scaled(W.CONFIGS["prefill"], T=8, d=1024, n_experts=64, inter=64, inter_shared=64,
                   dtype=torch.float32)
    c = W.make_centroids(cfg)
    n = c.norm(dim=1)
    R = 0.006 * math.sqrt(1024)
    srt = torch.sort(n, descending=True).values
    want = torch.tensor([R * (r + 1) ** -1.1 for r in range(64)])
    assert torch.allclose(srt, want, rtol=1e-5)


def test_w1_w3_share_one_buffer():
    # W1 and W3 are the two halves of one [2, E, I, d] buffer: w3 starts a fixed, 16-byte-multiple
    # distance after w1, the placement that lets the up-projection fetch both with one request
    for name in ("small", "mid"):
        cfg = W.scaled(W.CONFIGS[name], T=8, d=64, n_experts=4, inter=32, inter_shared=32)
        L = W.make_layer(cfg)
        for stack in (L["routed"], L["shared"]):
            w1, w3 = stack["w1"], stack["w3"]
            assert w1.is_contiguous() and w3.is_contiguous()
            gap = w3.data_ptr() - w1.data_ptr()
            assert gap == w1.numel() * w1.element_size() and gap % 16 == 0
            assert w1.untyped_storage().data_ptr() == w3.untyped_storage().data_ptr()
        # slices of experts keep the distance (expert-parallel ranks pass such slices)
        r = L["routed"]
        assert r["w3"][1:3].data_ptr() - r["w1"][1:3].data_ptr() == r["w1"].numel() * r["w1"].element_size()
