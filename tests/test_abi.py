"""The C-ABI library loads, exports every entry point include/moe.h declares, and rejects bad
arguments synchronously, before touching the GPU (CPU only: no compute call runs here)."""
import ctypes
import os
import re

import pytest

from fine_grained_mixture_route_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(moe.LIB_PATH):
        from fine_grained_mixture_route_b200 import build
        build.build()
    return moe.lib_handle()


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert {"moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward",
            "moe_workspace_bytes"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(moe.EXPORTED) == declared


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.moe_version()
    for s in range(6):
        assert lib.moe_status_string(s)
    assert lib.moe_status_string(99) == b"MOE_ERR_UNKNOWN"


def _shape(**kw):
    base = dict(T=256, d=7168, n_experts=256, inter=2048, top_k=8, n_shared=1, inter_shared=2048, has_bias=1,
                dtype=moe.MOE_BF16, gate_mode=0, routed_fmt=moe.FMT_NATIVE)
    base.update(kw)
    return moe.MoeShape(*[base[f] for f, _ in moe.MoeShape._fields_])


def test_workspace_bytes(lib):
    n = moe.workspace_bytes(_shape())
    S, d, I = 256 * 8, 7168, 2048
    # x_perm, h_r, Y (bf16) and the shared hidden states at least
    assert n >= 2 * (S * d + S * I + S * d + 256 * 2048)
    # ... plus the split-K router's fp32 partial logits (at most 148 CTAs x 128 tokens x N_m)
    assert n < 2 * (S * d + S * I + S * d + 256 * 2048) + 4 * 1024 * 1024 + 148 * 128 * 256 * 4
    assert moe.workspace_bytes(_shape(T=512)) > n
    assert moe.workspace_bytes(_shape(T=0)) > 0
    # fp32 layers keep no gathered copy of x
    assert moe.workspace_bytes(_shape(dtype=moe.MOE_F32)) < 2 * n
    for bad in (dict(top_k=0), dict(top_k=300), dict(n_experts=0), dict(d=0), dict(T=-1), dict(dtype=7),
                dict(n_experts=2048, top_k=8), dict(d=7170), dict(inter=2047), dict(top_k=33, n_experts=64),
                dict(has_bias=2), dict(n_shared=1, inter_shared=0), dict(gate_mode=3), dict(gate_mode=-1)):
        assert moe.workspace_bytes(_shape(**bad)) == 0, bad
    assert moe.workspace_bytes(_shape(d=7170, dtype=moe.MOE_F32)) > 0
    # e4m3 routed experts: h8 rows, per-token x codes and the per-row scale arrays on top (the
    # gathered x codes reuse x_perm)
    n8 = moe.workspace_bytes(_shape(routed_fmt=moe.FMT_E4M3))
    extra = S * I + 2 * 4 * S + 256 * d + 4 * 256
    assert extra <= n8 - n <= extra + 5 * 256
    for bad in (dict(routed_fmt=3), dict(routed_fmt=-1)):
        assert moe.workspace_bytes(_shape(**bad)) == 0, bad
    for unsupported in (dict(dtype=moe.MOE_F32), dict(d=7176), dict(inter=2056)):
        assert moe.workspace_bytes(_shape(routed_fmt=moe.FMT_E4M3, **unsupported)) == 0, unsupported


def test_launch_count(lib):
    # T=256: split-K router (scores + finish); 2048 slots grouped by one block (one launch, not three)
    assert moe.layer_launches(_shape()) == 8
    assert moe.layer_launches(_shape(T=16384)) == 9
    assert moe.layer_launches(_shape(T=16384, n_shared=0)) == 9
    assert moe.layer_launches(_shape(T=2048)) == 8     # 16384 slots: still one grouping block (split-K router)
    assert moe.layer_launches(_shape(T=2049)) == 10    # past 16384 slots: the three grouping passes
    assert moe.layer_launches(_shape(T=128, d=256, n_experts=16, inter=64, inter_shared=64, top_k=4,
                                     dtype=moe.MOE_F32)) == 6
    assert moe.layer_launches(_shape(routed_fmt=moe.FMT_E4M3)) == 10      # + x per token, hidden rows
    assert moe.layer_launches(_shape(T=0)) == 0
    assert moe.layer_launches(_shape(top_k=0)) == -1


def test_argument_errors_return_before_any_launch(lib):
    sh = _shape()
    fake = ctypes.c_void_p(1 << 40)            # never dereferenced: validation fails first
    n = moe.workspace_bytes(sh)
    w = moe.MoeWeights(fake.value, fake.value, fake.value, fake.value, fake.value, fake.value)
    S = ctypes.byref
    # null pointers
    assert lib.moe_route(S(sh), None, fake, None, fake, fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_forward(S(sh), fake, fake, None, None, S(w), fake, None, None, None, fake, n, None) == \
        moe.MOE_ERR_INVALID_ARG
    # bias pointers must match has_bias
    wnb = moe.MoeWeights(fake.value, None, fake.value, None, fake.value, None)
    assert lib.moe_expert_ffn(S(sh), fake, fake, fake, fake, S(wnb), fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    sh_nb = _shape(has_bias=0)
    assert lib.moe_expert_ffn(S(sh_nb), fake, fake, fake, fake, S(w), fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    # shared weights given for a layer without shared experts, and missing when needed
    sh0 = _shape(n_shared=0)
    assert lib.moe_combine(S(sh0), fake, S(w), fake, fake, fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(S(sh), fake, None, fake, fake, fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    # workspace too small, missing or misaligned
    assert lib.moe_route(S(sh), fake, fake, None, fake, fake, fake, n - 1, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_route(S(sh), fake, fake, None, fake, fake, None, n, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_route(S(sh), fake, fake, None, fake, fake, ctypes.c_void_p((1 << 40) + 8), n, None) == \
        moe.MOE_ERR_WORKSPACE
    # unsupported sizes
    assert lib.moe_route(S(_shape(d=7172)), fake, fake, None, fake, fake, fake, n, None) == moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_route(S(_shape(top_k=40, n_experts=64)), fake, fake, None, fake, fake, fake, n, None) == \
        moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_route(None, fake, fake, None, fake, fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_route(S(_shape(gate_mode=5)), fake, fake, None, fake, fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    # T == 0 is a valid no-op (returns before any CUDA call)
    sh_e = _shape(T=0)
    ne = moe.workspace_bytes(sh_e)
    assert lib.moe_route(S(sh_e), fake, fake, None, fake, fake, fake, ne, None) == moe.MOE_OK
    assert lib.moe_layer_forward(S(sh_e), fake, fake, None, S(w), S(w), fake, None, None, None, fake, ne, None) == moe.MOE_OK
    # ... also with the null data pointers of empty tensors for every per-token array
    assert lib.moe_route(S(sh_e), None, fake, None, None, None, fake, ne, None) == moe.MOE_OK
    assert lib.moe_expert_ffn(S(sh_e), None, fake, None, None, S(w), None, fake, ne, None) == moe.MOE_OK
    assert lib.moe_combine(S(sh_e), None, S(w), None, None, None, fake, ne, None) == moe.MOE_OK
    assert lib.moe_layer_forward(S(sh_e), None, fake, None, S(w), S(w), None, None, None, None, fake, ne, None) == \
        moe.MOE_OK
    # ... but the per-expert and weight arguments are still required
    assert lib.moe_route(S(sh_e), None, None, None, None, None, fake, ne, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_ffn(S(sh_e), None, None, None, None, S(w), None, fake, ne, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_ws_init(None, 0, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_check_device_error(None, 0, None, None) == moe.MOE_ERR_WORKSPACE
    # scales: required by e4m3 routed experts, refused elsewhere (native routed, shared)
    sh8 = _shape(routed_fmt=moe.FMT_E4M3)
    n8 = moe.workspace_bytes(sh8)
    w8 = moe.MoeWeights(*([fake.value] * 9))
    assert lib.moe_expert_ffn(S(sh8), fake, fake, fake, fake, S(w), fake, fake, n8, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_ffn(S(sh), fake, fake, fake, fake, S(w8), fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_forward(S(sh8), fake, fake, None, S(w8), S(w8), fake, None, None, None, fake, n8, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_forward(S(sh8), fake, fake, None, S(w8), S(w), fake, None, None, None, fake, n8 - 1, None) == \
        moe.MOE_ERR_WORKSPACE


def test_quantize_rows_argument_errors(lib):
    fake = ctypes.c_void_p(1 << 40)
    q = lib.moe_quantize_rows_e4m3
    assert q(fake, None, 10, 10, 12, fake, fake, fake, 4096, None) == moe.MOE_ERR_UNSUPPORTED   # width % 8
    assert q(fake, None, 11, 10, 16, fake, fake, fake, 4096, None) == moe.MOE_ERR_INVALID_ARG   # n_rows > src_rows
    assert q(fake, None, -1, 10, 16, fake, fake, fake, 4096, None) == moe.MOE_ERR_INVALID_ARG
    assert q(fake, None, 10, 10, 0, fake, fake, fake, 4096, None) == moe.MOE_ERR_INVALID_ARG
    assert q(fake, None, 10, 10, 16, fake, fake, None, 0, None) == moe.MOE_ERR_WORKSPACE
    assert q(None, None, 10, 10, 16, fake, fake, fake, 4096, None) == moe.MOE_ERR_INVALID_ARG
    assert q(fake, fake, 0, 10, 16, fake, fake, fake, 4096, None) == moe.MOE_OK                # no rows: no-op


def test_training_entry_points_validate(lib):
    fake = ctypes.c_void_p(1 << 40)
    S = ctypes.byref
    sh = _shape()
    assert moe.train_ctx_bytes(sh) > 0 and moe.backward_workspace_bytes(sh) > 0
    # ctx holds picks, grouping and the bf16 pre-activations a, g (routed and shared)
    Sl, I, T = 256 * 8, 2048, 256
    assert moe.train_ctx_bytes(sh) >= 2 * 2 * (Sl * I + T * 2048)
    for unsupported in (dict(dtype=moe.MOE_F32), dict(routed_fmt=moe.FMT_E4M3), dict(n_experts=512, top_k=8),
                        dict(n_experts=20, top_k=3), dict(d=7168 + 8), dict(inter=2048 + 16),
                        dict(inter_shared=2048 + 32)):
        assert moe.train_ctx_bytes(_shape(**unsupported)) == 0, unsupported
        assert moe.backward_workspace_bytes(_shape(**unsupported)) == 0, unsupported
    n, nb, nc = moe.workspace_bytes(sh), moe.backward_workspace_bytes(sh), moe.train_ctx_bytes(sh)
    w = moe.MoeWeights(*([fake.value] * 6))
    g = moe.MoeGrads(*([fake.value] * 6))
    f = lib.moe_layer_forward_train
    assert f(S(sh), fake, fake, None, S(w), S(w), fake, None, nc, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    assert f(S(sh), fake, fake, None, S(w), S(w), fake, fake, nc - 1, fake, n, None) == moe.MOE_ERR_WORKSPACE
    assert f(S(_shape(dtype=moe.MOE_F32)), fake, fake, None, S(w), S(w), fake, fake, nc, fake, n, None) == \
        moe.MOE_ERR_UNSUPPORTED
    b = lib.moe_layer_backward
    args = lambda **kw: [S(kw.get("sh", sh)), fake, fake, kw.get("rb", None), S(w), S(w), fake, fake,
                         kw.get("nc", nc), kw.get("dx", fake), fake, kw.get("drb", None), S(kw.get("g", g)),
                         S(kw.get("gs", g)), fake, kw.get("nb", nb), None]
    assert b(*args(nc=nc - 1)) == moe.MOE_ERR_WORKSPACE
    assert b(*args(nb=nb - 1)) == moe.MOE_ERR_WORKSPACE
    assert b(*args(drb=fake)) == moe.MOE_ERR_INVALID_ARG            # router-bias gradient without a bias
    assert b(*args(g=moe.MoeGrads(fake.value, None, fake.value, fake.value, fake.value, fake.value))) == \
        moe.MOE_ERR_INVALID_ARG                                      # bias gradient pointers must match has_bias
    # gradients, dx and dcentroids take 16-byte vector and tensor-memory-access stores
    odd = ctypes.c_void_p((1 << 40) + 8)
    assert b(*args()) not in (moe.MOE_OK, moe.MOE_ERR_INVALID_ARG)   # aligned: past validation (no device here)
    assert b(*args(dx=odd)) == moe.MOE_ERR_INVALID_ARG
    for i in range(6):
        ptrs = [fake.value] * 6
        ptrs[i] = odd.value
        assert b(*args(g=moe.MoeGrads(*ptrs))) == moe.MOE_ERR_INVALID_ARG, i
        assert b(*args(gs=moe.MoeGrads(*ptrs))) == moe.MOE_ERR_INVALID_ARG, i
    sh2 = _shape(gate_mode=2)
    assert b(*args(sh=sh2, rb=fake, drb=fake, nc=moe.train_ctx_bytes(sh2), nb=moe.backward_workspace_bytes(sh2))) \
        == moe.MOE_ERR_INVALID_ARG                                   # gate mode 2: the bias only selects
    sh0 = _shape(T=0)
    assert b(*args(sh=sh0, nc=moe.train_ctx_bytes(sh0), nb=moe.backward_workspace_bytes(sh0))) == moe.MOE_OK
    a0 = args(sh=sh0, nc=moe.train_ctx_bytes(sh0), nb=moe.backward_workspace_bytes(sh0))
    a0[1], a0[6], a0[9] = None, None, None                          # x, dout, dx of an empty batch
    assert b(*a0) == moe.MOE_OK


def test_balance_stats_validate(lib):
    fake = ctypes.c_void_p(1 << 40)
    S = ctypes.byref
    sh = _shape()
    n = lib.moe_balance_workspace_bytes(S(sh))
    assert n >= 256 * 256 * 4                                   # the T x N_m score matrix at least
    assert lib.moe_balance_workspace_bytes(S(_shape(dtype=moe.MOE_F32))) == 0
    assert lib.moe_balance_workspace_bytes(S(_shape(n_experts=512))) == 0
    q = lib.moe_balance_stats
    assert q(S(sh), fake, fake, None, fake, 3, fake, fake, fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG   # 3 !| 256
    assert q(S(sh), fake, fake, None, fake, 0, fake, fake, fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    assert q(S(sh), fake, fake, None, None, 4, fake, fake, fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    assert q(S(sh), fake, fake, None, fake, 4, fake, fake, fake, fake, n - 1, None) == moe.MOE_ERR_WORKSPACE
    assert q(S(_shape(dtype=moe.MOE_F32)), fake, fake, None, fake, 4, fake, fake, fake, fake, n, None) == \
        moe.MOE_ERR_UNSUPPORTED


def test_segment_ids_and_wait_selftest_argument_errors(lib):
    """The expert-parallel segment-id call and the bounded-wait self-test reject bad arguments
    before any launch."""
    fake = ctypes.c_void_p(1 << 40)
    ws = ctypes.c_void_p(1 << 41)
    assert lib.moe_segment_ids(fake, 0, 4, 10, fake, ws, 256, None) == moe.MOE_ERR_INVALID_ARG      # no segments
    assert lib.moe_segment_ids(fake, 8, 0, 10, fake, ws, 256, None) == moe.MOE_ERR_INVALID_ARG      # modulo 0
    assert lib.moe_segment_ids(fake, 8, 4, -1, fake, ws, 256, None) == moe.MOE_ERR_INVALID_ARG      # negative rows
    assert lib.moe_segment_ids(fake, 4097, 4, 10, fake, ws, 256, None) == moe.MOE_ERR_UNSUPPORTED   # > 4096 segments
    assert lib.moe_segment_ids(fake, 8, 4, 10, fake, None, 256, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_segment_ids(fake, 8, 4, 10, fake, ws, 255, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_segment_ids(fake, 8, 4, 0, None, ws, 256, None) == moe.MOE_OK                  # nothing to do
    assert lib.moe_segment_ids(None, 8, 4, 10, fake, ws, 256, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_wait_timeout(999, None, ws, 256, None) == moe.MOE_ERR_INVALID_ARG        # < 1 us
    assert lib.moe_selftest_wait_timeout(10**10 + 1, None, ws, 256, None) == moe.MOE_ERR_INVALID_ARG  # > 10 s
    assert lib.moe_selftest_wait_timeout(10**6, None, None, 256, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_selftest_wait_timeout(10**6, ctypes.c_void_p((1 << 40) + 4), ws, 256, None) == \
        moe.MOE_ERR_INVALID_ARG                                                                       # misaligned out


def test_mxfp8_format_validates(lib):
    """Block-scaled FP8 routed experts: the layer needs the scale bytes (and no per-row scales),
    every other stack refuses them, they must be 16-byte aligned; the scale-array size and the
    quantiser's argument checks follow include/moe.h."""
    fake = ctypes.c_void_p(1 << 40)
    S = ctypes.byref
    shm = _shape(routed_fmt=moe.FMT_MXFP8)
    nm = moe.workspace_bytes(shm)
    # on top of the e4m3 workspace: x's run scales per token, and the tiled A-side scales of both
    # GEMMs (one 512-byte block per (128-row block, 128-input chunk); at most S/128 + E blocks)
    T, d, I, E, slots = 256, 7168, 2048, 256, 256 * 8
    al = lambda n: (n + 255) // 256 * 256
    extra = al(T * d // 32) + al((slots // 128 + E) * (d // 128) * 512) + al((slots // 128 + E) * (I // 128) * 512)
    assert nm - moe.workspace_bytes(_shape(routed_fmt=moe.FMT_E4M3)) == extra
    assert moe.layer_launches(shm) == moe.layer_launches(_shape(routed_fmt=moe.FMT_E4M3)) == 10
    for unsupported in (dict(dtype=moe.MOE_F32), dict(d=7176), dict(inter=2056)):
        assert moe.workspace_bytes(_shape(routed_fmt=moe.FMT_MXFP8, **unsupported)) == 0, unsupported
    f = fake.value
    w = moe.MoeWeights(f, f, f, f, f, f)
    w8 = moe.MoeWeights(f, f, f, f, f, f, f, f, f)
    wm = moe.MoeWeights(f, f, f, f, f, f, None, None, None, f, f)
    wboth = moe.MoeWeights(*([f] * 11))
    wmis = moe.MoeWeights(f, f, f, f, f, f, None, None, None, f + 8, f)
    ffn = lib.moe_expert_ffn
    for bad in (w, w8, wboth, wmis):
        assert ffn(S(shm), fake, fake, fake, fake, S(bad), fake, fake, nm, None) == moe.MOE_ERR_INVALID_ARG
    sh8, n8 = _shape(routed_fmt=moe.FMT_E4M3), moe.workspace_bytes(_shape(routed_fmt=moe.FMT_E4M3))
    assert ffn(S(sh8), fake, fake, fake, fake, S(wboth), fake, fake, n8, None) == moe.MOE_ERR_INVALID_ARG
    sh, n = _shape(), moe.workspace_bytes(_shape())
    assert ffn(S(sh), fake, fake, fake, fake, S(wm), fake, fake, n, None) == moe.MOE_ERR_INVALID_ARG
    # shared experts stay bf16: scale bytes on the shared stack are refused
    assert lib.moe_layer_forward(S(shm), fake, fake, None, S(wm), S(wm), fake, None, None, None, fake, nm, None) == \
        moe.MOE_ERR_INVALID_ARG
    # scale-array sizes: 1 KB per (expert, row group, 128-input chunk)
    sb = lib.moe_mx_scale_bytes
    assert sb(moe.MX_UP, 256, 2048, 7168) == 256 * 16 * 56 * 1024
    assert sb(moe.MX_DOWN, 256, 7168, 2048) == 256 * 28 * 16 * 1024
    assert sb(moe.MX_UP, 3, 200, 208) == 3 * 2 * 2 * 1024
    assert sb(moe.MX_DOWN, 1, 300, 16) == 2 * 1 * 1024
    assert sb(2, 1, 1, 1) == 0 and sb(moe.MX_UP, 0, 1, 1) == 0 and sb(moe.MX_UP, 1, 1, 0) == 0
    q = lib.moe_quantize_weights_mx
    assert q(2, fake, None, 1, 32, 32, fake, None, fake, None) == moe.MOE_ERR_INVALID_ARG          # kind
    assert q(moe.MX_DOWN, fake, fake, 1, 32, 32, fake, fake, fake, None) == moe.MOE_ERR_INVALID_ARG  # one matrix
    assert q(moe.MX_UP, fake, None, 1, 32, 32, fake, None, fake, None) == moe.MOE_ERR_INVALID_ARG    # w3 missing
    assert q(moe.MX_DOWN, fake, None, 1, 32, 24, fake, None, fake, None) == moe.MOE_ERR_UNSUPPORTED  # K % 16
    assert q(moe.MX_DOWN, fake, None, 0, 32, 32, fake, None, fake, None) == moe.MOE_ERR_INVALID_ARG
    assert q(moe.MX_DOWN, None, None, 1, 32, 32, fake, None, fake, None) == moe.MOE_ERR_INVALID_ARG
    assert q(moe.MX_DOWN, fake, None, 1, 32, 32, fake, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert q(moe.MX_DOWN, ctypes.c_void_p(f + 8), None, 1, 32, 32, fake, None, fake, None) == moe.MOE_ERR_INVALID_ARG
