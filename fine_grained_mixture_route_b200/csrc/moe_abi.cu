// The C ABI of include/moe.h: argument validation, workspace layout, and the launch
// sequence of each entry point on the caller's stream.  No allocation, no host sync (except
// in moe_check_device_error), no exceptions.
#include <cstring>

#include "common.cuh"
#include "abi_checks.h"
#include "launch.h"

#define MOE_EXPORT __attribute__((visibility("default")))

namespace moe {
namespace {

size_t al(size_t x) { return (x + 255) & ~(size_t)255; }

struct Layout {
    size_t err, hist, rpart, sout, ts1, ts2, idx, gate, counts, offsets, stok, sgate, slot_of, xperm, hr, hs, y;
    size_t xs, h8, hsc;    // e4m3 routed experts: row scales of x8 (in xperm), h8 rows and their scales
    size_t x8t, xst;       // e4m3: x quantised once per token, and its scales
    size_t xsf, sfa1, sfa2;  // block-scaled: x's run scales per token; GEMM1's and GEMM2's tiled A scales
    size_t total;
};

Layout layout(const Dims& D) {
    Layout L;
    const size_t S = (size_t)D.slots();
    const size_t esz = D.bf16 ? 2 : 4;
    const size_t nblk = (size_t)permute_blocks(D);
    size_t o = 0;
    L.err = o; o += 256;
    L.hist = o; o += al((nblk ? nblk : 1) * D.E * 4);
    L.rpart = o; o += al(router_partial_bytes(D));
    L.sout = o; o += (D.bf16 && D.Ks > 0) ? al((size_t)D.T * D.d * 4) : 0;
    L.ts1 = o; o += al((size_t)(D.E + D.Ks + 1) * 4);
    L.ts2 = o; o += al((size_t)(D.E + 1) * 4);
    L.idx = o; o += al(S * 4);
    L.gate = o; o += al(S * 4);
    L.counts = o; o += al((size_t)D.E * 4);
    L.offsets = o; o += al((size_t)(D.E + 1) * 4);
    L.stok = o; o += al(S * 4);
    L.sgate = o; o += al(S * 4);
    L.slot_of = o; o += al(S * 4);
    L.xperm = o; o += D.bf16 ? al(S * D.d * esz) : 0;
    L.hr = o; o += al(S * D.I * esz);
    L.hs = o; o += al((size_t)D.Ks * D.T * (D.Ks ? D.Is : 0) * esz);
    L.y = o; o += al(S * D.d * esz);
    L.xs = o; o += D.q8 ? al(S * 4) : 0;
    L.h8 = o; o += D.q8 ? al(S * D.I) : 0;
    L.hsc = o; o += D.q8 ? al(S * 4) : 0;
    L.x8t = o; o += D.q8 ? al((size_t)D.T * D.d) : 0;
    L.xst = o; o += D.q8 ? al((size_t)D.T * 4) : 0;
    L.xsf = o; o += D.mx ? al((size_t)D.T * ((D.d + 31) / 32)) : 0;
    L.sfa1 = o; o += D.mx ? al(mx_act_scale_bytes(D.slots(), D.E, D.d)) : 0;
    L.sfa2 = o; o += D.mx ? al(mx_act_scale_bytes(D.slots(), D.E, D.I)) : 0;
    L.total = o;
    return L;
}

// Training context: what moe_layer_forward_train keeps for moe_layer_backward.
struct CtxLayout {
    size_t idx, gate, counts, offsets, stok, sgate, slot_of, a, g, as, gs, total;
};
CtxLayout ctx_layout(const Dims& D) {
    CtxLayout C;
    const size_t S = (size_t)D.slots();
    size_t o = 0;
    C.idx = o; o += al(S * 4);
    C.gate = o; o += al(S * 4);
    C.counts = o; o += al((size_t)D.E * 4);
    C.offsets = o; o += al((size_t)(D.E + 1) * 4);
    C.stok = o; o += al(S * 4);
    C.sgate = o; o += al(S * 4);
    C.slot_of = o; o += al(S * 4);
    C.a = o; o += al(S * D.I * 2);
    C.g = o; o += al(S * D.I * 2);
    C.as = o; o += al((size_t)D.Ks * D.T * (D.Ks ? D.Is : 0) * 2);
    C.gs = o; o += al((size_t)D.Ks * D.T * (D.Ks ? D.Is : 0) * 2);
    C.total = o;
    return C;
}

// Backward workspace.
struct BwdLayout {
    size_t err, offs_pad, ts_dh, ts_dx, dout_pad, x_pad, gate_pad, b2dot, z, dgate_part, dag, hg, dag_s, hg_s, dz,
        dz_bf16, dx_slot, base, cpart, total;
    long long S_pad_max;
    int n_parts;
};
BwdLayout bwd_layout(const Dims& D) {
    BwdLayout B;
    const size_t S = (size_t)D.slots();
    B.S_pad_max = (long long)S + 64LL * D.E;
    const size_t Sp = (size_t)B.S_pad_max;
    const size_t Is = D.Ks ? D.Is : 0;
    B.n_parts = 2 * ((D.I + 255) / 256);
    size_t o = 0;
    B.err = o; o += 256;
    B.offs_pad = o; o += al((size_t)(D.E + 1) * 4);
    B.ts_dh = o; o += al((size_t)(D.E + D.Ks + 1) * 4);
    B.ts_dx = o; o += al((size_t)(D.E + 1) * 4);
    B.dout_pad = o; o += al(Sp * D.d * 2);
    B.x_pad = o; o += al(Sp * (D.d + 64) * 2);           // + the bias-gradient column block
    B.gate_pad = o; o += al(Sp * 4);
    B.b2dot = o; o += al(S * 4);
    B.z = o; o += al((size_t)D.T * D.E * 4);
    B.dgate_part = o; o += al(S * B.n_parts * 4);
    B.dag = o; o += al(Sp * 2 * D.I * 2);
    B.hg = o; o += al(Sp * (D.I + 64) * 2);
    B.dag_s = o; o += al((size_t)D.Ks * D.T * 2 * Is * 2);
    B.hg_s = o; o += al((size_t)D.Ks * D.T * (D.Ks ? Is + 64 : 0) * 2);
    B.dz = o; o += al((size_t)D.T * D.E * 4);
    B.dz_bf16 = o; o += al((size_t)D.T * D.E * 2);
    B.dx_slot = o; o += al(S * D.d * 2);
    B.base = o; o += al((size_t)D.T * D.d * 4);
    B.cpart = o; o += al((size_t)(D.Ks * 2 * Is + D.E) * ((D.T + 255) / 256) * 4);   // column-sum partials
    B.total = o;
    return B;
}

}  // namespace

// Shape and device checks shared with the allocation-free grouping entry point (abi_checks.h).
moe_status_t to_dims(const moe_shape_t* s, Dims* D) {
    if (!s) return MOE_ERR_INVALID_ARG;
    if (s->dtype != MOE_F32 && s->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (s->T < 0 || s->d < 1 || s->n_experts < 1 || s->inter < 1 || s->top_k < 1 || s->n_shared < 0)
        return MOE_ERR_INVALID_ARG;
    if (s->top_k > s->n_experts) return MOE_ERR_INVALID_ARG;
    if (s->n_shared > 0 && s->inter_shared < 1) return MOE_ERR_INVALID_ARG;
    if (s->has_bias != 0 && s->has_bias != 1) return MOE_ERR_INVALID_ARG;
    if (s->gate_mode < MOE_GATE_SOFTMAX_TOPK || s->gate_mode > MOE_GATE_SIGMOID_BIAS) return MOE_ERR_INVALID_ARG;
    if ((long long)s->T * s->top_k >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
    if (s->n_experts > 1024 || s->top_k > 32 || s->n_shared > 16) return MOE_ERR_UNSUPPORTED;
    if (s->dtype == MOE_BF16) {
        if (s->d % 8 || s->inter % 8 || (s->n_shared > 0 && s->inter_shared % 8)) return MOE_ERR_UNSUPPORTED;
    }
    if (s->routed_fmt != MOE_FMT_NATIVE && s->routed_fmt != MOE_FMT_E4M3 && s->routed_fmt != MOE_FMT_MXFP8)
        return MOE_ERR_INVALID_ARG;
    if (s->routed_fmt != MOE_FMT_NATIVE && (s->dtype != MOE_BF16 || s->d % 16 || s->inter % 16))
        return MOE_ERR_UNSUPPORTED;
    D->T = s->T; D->d = s->d; D->E = s->n_experts; D->I = s->inter; D->k = s->top_k;
    D->Ks = s->n_shared; D->Is = s->n_shared > 0 ? s->inter_shared : 0;
    D->bias = s->has_bias != 0; D->bf16 = s->dtype == MOE_BF16;
    D->gate_mode = s->gate_mode;
    D->q8 = s->routed_fmt != MOE_FMT_NATIVE;
    D->mx = s->routed_fmt == MOE_FMT_MXFP8;
    return MOE_OK;
}

moe_status_t check_ws(const Dims& D, void* ws, size_t ws_bytes) {
    if (!ws || ws_bytes < layout(D).total || ((uintptr_t)ws & 15u)) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

// The scale arrays a stack carries follow its format: the routed experts of an MOE_FMT_E4M3
// layer carry s1, s3, s2 (and no scale bytes), those of an MOE_FMT_MXFP8 layer sf13 and sf2 (and
// no per-channel scales); every other stack (native routed experts, shared experts) carries none.
moe_status_t check_weights(const Dims& D, const moe_ffn_weights_t* w, bool routed = false) {
    if (!w || !w->w1 || !w->w3 || !w->w2) return MOE_ERR_INVALID_ARG;
    const bool b = w->b1 && w->b3 && w->b2;
    const bool none = !w->b1 && !w->b3 && !w->b2;
    if (D.bias ? !b : !none) return MOE_ERR_INVALID_ARG;
    const bool sc = w->s1 && w->s3 && w->s2, nosc = !w->s1 && !w->s3 && !w->s2;
    const bool sf = w->sf13 && w->sf2, nosf = !w->sf13 && !w->sf2;
    const bool e4m3 = routed && D.q8 && !D.mx, mx = routed && D.mx;
    if (e4m3 ? !sc : !nosc) return MOE_ERR_INVALID_ARG;
    if (mx ? !sf : !nosf) return MOE_ERR_INVALID_ARG;
    if (mx && (((uintptr_t)w->sf13 | (uintptr_t)w->sf2) & 15u)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// Layers the training path (forward_train + backward) handles: bf16, native routed weights, a
// tensor-core router (it recomputes the logits), and d, inter, inter_shared multiples of 64.
moe_status_t check_train(const Dims& D) {
    if (!D.bf16 || D.q8 || !tc_router_supported(D)) return MOE_ERR_UNSUPPORTED;
    if (D.d % 64 || D.I % 64 || (D.Ks > 0 && D.Is % 64)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status_t check_device() {
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (major != 10) return MOE_ERR_UNSUPPORTED;   // built for sm_100a only
    return MOE_OK;
}

namespace {

#define MOE_TRY(expr)                              \
    do {                                           \
        moe_status_t _s = (expr);                  \
        if (_s != MOE_OK) return _s;               \
    } while (0)
#define MOE_CUDA(expr)                             \
    do {                                           \
        if ((expr) != cudaSuccess) return MOE_ERR_CUDA; \
    } while (0)

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

FfnWeights to_ffn(const moe_ffn_weights_t* w) {
    FfnWeights f = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
    if (w) {
        f.w1 = w->w1; f.b1 = w->b1; f.w3 = w->w3; f.b3 = w->b3; f.w2 = w->w2; f.b2 = w->b2;
        f.s1 = w->s1; f.s3 = w->s3; f.s2 = w->s2;
        f.sf13 = w->sf13; f.sf2 = w->sf2;
    }
    return f;
}

// e4m3 routed experts: x quantised once per token, then its code rows (and scales) gathered
// into expert order for the GEMM1 A operand.
// With the slot map at hand (the fused forward) the code rows are written in token order
// instead: each token's codes are read once and stored at its k slot positions.
// Block-scaled (D.mx): x quantised in runs of 32; the run scales go to GEMM1's tiled A-side
// layout by grouped position (needs the tile table ts1).
moe_status_t quant_gather_x(const Dims& D, const Layout& L, void* ws, const void* x, const int32_t* stok,
                            const int32_t* offsets, const int32_t* ts1, uint32_t* err, cudaStream_t st,
                            const int32_t* slot_of = nullptr) {
    uint8_t* x8t = at<uint8_t>(ws, L.x8t);
    float* xst = D.mx ? nullptr : at<float>(ws, L.xst);
    float* xs = D.mx ? nullptr : at<float>(ws, L.xs);
    if (D.mx) MOE_CUDA(launch_quant_rows_mx(x, D.T, D.d, x8t, at<uint8_t>(ws, L.xsf), st));
    else MOE_CUDA(launch_quant_rows(x, nullptr, D.T, D.T, D.d, x8t, xst, err, st));
    if (slot_of)
        MOE_CUDA(launch_scatter_code_rows(x8t, xst, slot_of, D.T, D.k, D.slots(), D.d, at<uint8_t>(ws, L.xperm), xs,
                                          err, st));
    else
        MOE_CUDA(launch_gather_code_rows(x8t, xst, stok, D.slots(), D.T, D.d, at<uint8_t>(ws, L.xperm), xs, err, st));
    if (D.mx)
        MOE_CUDA(launch_scatter_sf_tiled(at<uint8_t>(ws, L.xsf), D.T, D.d, stok, offsets, ts1, D.E, D.slots(), D.I,
                                         at<uint8_t>(ws, L.sfa1), err, st));
    return MOE_OK;
}

// Block-scaled activations: GEMM1 reads sfa1 and writes the hidden codes and sfa2; GEMM2 reads sfa2.
MxAct mx_gemm1(const Layout& L, void* ws) {
    MxAct m;
    m.sfa = at<uint8_t>(ws, L.sfa1);
    m.h8 = at<uint8_t>(ws, L.h8);
    m.sfh = at<uint8_t>(ws, L.sfa2);
    return m;
}
MxAct mx_gemm2(const Layout& L, void* ws) {
    MxAct m;
    m.sfa = at<uint8_t>(ws, L.sfa2);
    return m;
}

moe_status_t do_route(const Dims& D, const void* x, const void* c, const float* bias, int32_t* idx, float* gate,
                      float* partial, uint32_t* err, cudaStream_t st) {
    if (D.T == 0) return MOE_OK;
    if (tc_router_supported(D)) MOE_CUDA(launch_tc_router(D, x, c, bias, idx, gate, partial, err, st));
    else MOE_CUDA(launch_router_simt(D, x, c, bias, idx, gate, st));
    return MOE_OK;
}

// routed experts: y_sorted = gate * FFN_e(x[sorted_token])
moe_status_t do_expert_ffn(const Dims& D, const Layout& L, void* ws, const void* x, const int32_t* offsets,
                           const int32_t* stok, const float* sgate, const FfnWeights& R, void* y, bool plan_done,
                           cudaStream_t st) {
    uint32_t* err = at<uint32_t>(ws, L.err);
    int32_t* ts1 = at<int32_t>(ws, L.ts1);
    int32_t* ts2 = at<int32_t>(ws, L.ts2);
    if (!plan_done) MOE_CUDA(launch_plan(D, offsets, ts1, ts2, err, st));
    if (D.q8) {
        uint8_t* x8 = at<uint8_t>(ws, L.xperm);
        float* xs = D.mx ? nullptr : at<float>(ws, L.xs);
        MOE_TRY(quant_gather_x(D, L, ws, x, stok, offsets, ts1, err, st));
        FfnWeights none = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
        const MxAct m1 = mx_gemm1(L, ws), m2 = mx_gemm2(L, ws);
        MOE_CUDA(launch_tc_gemm1_q8(D, x, x8, xs, offsets, ts1, R, none, at<void>(ws, L.hr), nullptr, D.E, err, st,
                                    D.mx ? &m1 : nullptr));
        uint8_t* h8 = at<uint8_t>(ws, L.h8);
        float* hsc = D.mx ? nullptr : at<float>(ws, L.hsc);
        if (!D.mx)   // block-scaled: GEMM1 already wrote the hidden rows as codes with their run scales
            MOE_CUDA(launch_quant_rows(at<void>(ws, L.hr), nullptr, D.slots(), (int)D.slots(), D.I, h8, hsc, err, st));
        MOE_CUDA(launch_tc_gemm2_routed_q8(D, offsets, ts2, sgate, R, h8, hsc, y, nullptr, nullptr, nullptr, err, st,
                                           D.mx ? &m2 : nullptr));
    } else if (D.bf16) {
        void* xp = at<void>(ws, L.xperm);
        MOE_CUDA(launch_gather(D, x, stok, xp, err, st));
        FfnWeights none = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
        MOE_CUDA(launch_tc_gemm1(D, x, xp, offsets, ts1, R, none, at<void>(ws, L.hr), nullptr, 0, D.E, err, st));
        MOE_CUDA(launch_tc_gemm2_routed(D, offsets, ts2, sgate, R, at<void>(ws, L.hr), y, nullptr, nullptr, nullptr,
                                        err, st));
    } else {
        FfnWeights none = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
        MOE_CUDA(launch_simt_gemm1(D, x, offsets, stok, R, none, at<void>(ws, L.hr), nullptr, 0, D.E, err, st));
        MOE_CUDA(launch_simt_gemm2_routed(D, offsets, sgate, R, at<void>(ws, L.hr), y, err, st));
    }
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

MOE_EXPORT size_t moe_workspace_bytes(const moe_shape_t* shape) {
    Dims D;
    if (to_dims(shape, &D) != MOE_OK) return 0;
    return layout(D).total;
}

MOE_EXPORT const char* moe_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null pointer, size out of range or bias mismatch";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: valid layer outside what these kernels handle";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or kernel launch failed";
        case MOE_ERR_INTERNAL: return "MOE_ERR_INTERNAL: a kernel flagged an error";
    }
    return "MOE_ERR_UNKNOWN";
}

MOE_EXPORT int32_t moe_layer_launches(const moe_shape_t* shape) {
    Dims D;
    if (to_dims(shape, &D) != MOE_OK) return -1;
    if (D.T == 0) return 0;
    int n = 0;
    if (tc_router_supported(D)) n += router_splits(D) > 1 ? 2 : 1;   // scores (+ split-K finish)
    else n += 1;
    n += permute_small(D) ? 1 : 3;                                  // histogram, scan, scatter (one block if small)
    n += 1;                                                         // tile tables
    if (D.bf16) n += 1;                                             // row gather (+ e4m3 quantisation)
    n += 3;                                   // GEMM1, GEMM2 (routed + shared tiles), combine
    if (D.q8) n += 2;   // per-token x quantisation, hidden-row quantisation (block-scaled: scale scatter)
    return n;
}

MOE_EXPORT const char* moe_version(void) { return "moe_b200 0.1 sm_100a"; }

MOE_EXPORT moe_status_t moe_ws_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (!ws || ws_bytes < 256) return MOE_ERR_WORKSPACE;
    if (cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

MOE_EXPORT moe_status_t moe_check_device_error(void* ws, size_t ws_bytes, moe_stream_t stream, uint32_t* detail) {
    if (!ws || ws_bytes < 256) return MOE_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t h = 0;
    if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    if (detail) *detail = h;
    if (h) {
        if (cudaMemsetAsync(ws, 0, sizeof(h), st) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_ERR_INTERNAL;
    }
    return MOE_OK;
}

MOE_EXPORT moe_status_t moe_route(const moe_shape_t* shape, const void* x, const void* centroids,
                                  const float* router_bias, int32_t* topk_idx, float* topk_gate, void* ws,
                                  size_t ws_bytes, moe_stream_t stream) {
    Dims D;
    MOE_TRY(to_dims(shape, &D));
    if (!centroids || (D.T > 0 && (!x || !topk_idx || !topk_gate))) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ws(D, ws, ws_bytes));
    if (D.T == 0) return MOE_OK;
    MOE_TRY(check_device());
    cudaGetLastError();
    const Layout L = layout(D);
    return do_route(D, x, centroids, router_bias, topk_idx, topk_gate, at<float>(ws, L.rpart),
                    at<uint32_t>(ws, L.err), (cudaStream_t)stream);
}

MOE_EXPORT moe_status_t moe_permute(const moe_shape_t* shape, const int32_t* topk_idx, const float* topk_gate,
                                    int32_t* counts, int32_t* offsets, int32_t* sorted_token, float* sorted_gate,
                                    int32_t* slot_of, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Dims D;
    MOE_TRY(to_dims(shape, &D));
    if (!counts || !offsets || (D.T > 0 && (!topk_idx || !topk_gate || !sorted_token || !sorted_gate || !slot_of)))
        return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ws(D, ws, ws_bytes));
    MOE_TRY(check_device());
    cudaGetLastError();
    const Layout L = layout(D);
    MOE_CUDA(launch_permute(D, topk_idx, topk_gate, counts, offsets, sorted_token, sorted_gate, slot_of,
                            at<int32_t>(ws, L.hist), at<uint32_t>(ws, L.err), (cudaStream_t)stream));
    return MOE_OK;
}

MOE_EXPORT moe_status_t moe_expert_ffn(const moe_shape_t* shape, const void* x, const int32_t* offsets,
                                       const int32_t* sorted_token, const float* sorted_gate,
                                       const moe_ffn_weights_t* routed, void* y_sorted, void* ws, size_t ws_bytes,
                                       moe_stream_t stream) {
    Dims D;
    MOE_TRY(to_dims(shape, &D));
    if (!offsets || (D.T > 0 && (!x || !sorted_token || !y_sorted))) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_weights(D, routed, true));
    MOE_TRY(check_ws(D, ws, ws_bytes));
    if (D.T == 0) return MOE_OK;
    MOE_TRY(check_device());
    cudaGetLastError();
    const Layout L = layout(D);
    return do_expert_ffn(D, L, ws, x, offsets, sorted_token, sorted_gate, to_ffn(routed), y_sorted, false,
                         (cudaStream_t)stream);
}

MOE_EXPORT moe_status_t moe_combine(const moe_shape_t* shape, const void* x, const moe_ffn_weights_t* shared,
                                    const void* y_sorted, const int32_t* slot_of, void* out, void* ws,
                                    size_t ws_bytes, moe_stream_t stream) {
    Dims D;
    MOE_TRY(to_dims(shape, &D));
    if (D.T > 0 && (!y_sorted || !slot_of || !out)) return MOE_ERR_INVALID_ARG;
    if (D.Ks > 0) {
        if (D.T > 0 && !x) return MOE_ERR_INVALID_ARG;
        MOE_TRY(check_weights(D, shared));
    } else if (shared) {
        return MOE_ERR_INVALID_ARG;
    }
    MOE_TRY(check_ws(D, ws, ws_bytes));
    if (D.T == 0) return MOE_OK;
    MOE_TRY(check_device());
    cudaGetLastError();
    const Layout L = layout(D);
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t* err = at<uint32_t>(ws, L.err);
    if (D.Ks == 0) {
        MOE_CUDA(launch_combine(D, y_sorted, slot_of, nullptr, out, err, st));
        return MOE_OK;
    }
    const FfnWeights Sh = to_ffn(shared);
    const FfnWeights none = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
    void* hs = at<void>(ws, L.hs);
    if (D.bf16) {
        int32_t* ts1 = at<int32_t>(ws, L.ts1);
        MOE_CUDA(launch_plan(D, nullptr, ts1, at<int32_t>(ws, L.ts2), err, st));
        MOE_CUDA(launch_tc_gemm1(D, x, nullptr, nullptr, ts1, none, Sh, nullptr, hs, D.E, D.E + D.Ks, err, st));
        float* sout = at<float>(ws, L.sout);
        MOE_CUDA(launch_tc_gemm2_shared(D, Sh, hs, sout, err, st));
        MOE_CUDA(launch_combine(D, y_sorted, slot_of, sout, out, err, st));
    } else {
        MOE_CUDA(launch_simt_gemm1(D, x, nullptr, nullptr, none, Sh, nullptr, hs, D.E, D.E + D.Ks, err, st));
        MOE_CUDA(launch_simt_gemm2_shared(D, Sh, hs, y_sorted, slot_of, out, err, st));
    }
    return MOE_OK;
}

MOE_EXPORT moe_status_t moe_quantize_rows_e4m3(const void* src, const int32_t* row_of, int64_t n_rows,
                                               int32_t src_rows, int32_t width, uint8_t* dst, float* scale, void* ws,
                                               size_t ws_bytes, moe_stream_t stream) {
    if (n_rows < 0 || src_rows < 0 || width < 1 || n_rows >= (1LL << 31)) return MOE_ERR_INVALID_ARG;
    if (!row_of && n_rows > src_rows) return MOE_ERR_INVALID_ARG;
    if (width % 8) return MOE_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < 256 || ((uintptr_t)ws & 15u)) return MOE_ERR_WORKSPACE;
    if (n_rows == 0) return MOE_OK;
    if (!src || !dst || !scale) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_device());
    cudaGetLastError();
    MOE_CUDA(launch_quant_rows(src, row_of, n_rows, src_rows, width, dst, scale, static_cast<uint32_t*>(ws),
                               (cudaStream_t)stream));
    return MOE_OK;
}

MOE_EXPORT size_t moe_mx_scale_bytes(int32_t kind, int32_t n_experts, int32_t rows, int32_t K) {
    if ((kind != MOE_MX_UP && kind != MOE_MX_DOWN) || n_experts < 1 || rows < 1 || K < 1) return 0;
    return mx_scale_bytes(kind, n_experts, rows, K);
}

MOE_EXPORT moe_status_t moe_quantize_weights_mx(int32_t kind, const void* w_a, const void* w_b, int32_t n_experts,
                                                int32_t rows, int32_t K, uint8_t* codes_a, uint8_t* codes_b,
                                                uint8_t* sf, moe_stream_t stream) {
    if (kind != MOE_MX_UP && kind != MOE_MX_DOWN) return MOE_ERR_INVALID_ARG;
    if (n_experts < 1 || rows < 1 || K < 1 || (long long)n_experts * rows >= (1LL << 31)) return MOE_ERR_INVALID_ARG;
    if (!w_a || !codes_a || !sf) return MOE_ERR_INVALID_ARG;
    if (kind == MOE_MX_UP ? (!w_b || !codes_b) : (w_b || codes_b)) return MOE_ERR_INVALID_ARG;
    if (K % 16) return MOE_ERR_UNSUPPORTED;
    const uintptr_t al = (uintptr_t)w_a | (uintptr_t)w_b | (uintptr_t)codes_a | (uintptr_t)codes_b | (uintptr_t)sf;
    if (al & 15u) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_device());
    cudaGetLastError();
    const cudaStream_t st = (cudaStream_t)stream;
    MOE_CUDA(cudaMemsetAsync(sf, 127, mx_scale_bytes(kind, n_experts, rows, K), st));
    MOE_CUDA(launch_quant_weights_mx(kind, w_a, 0, n_experts, rows, K, codes_a, sf, st));
    if (kind == MOE_MX_UP) MOE_CUDA(launch_quant_weights_mx(kind, w_b, 1, n_experts, rows, K, codes_b, sf, st));
    return MOE_OK;
}

}  // extern "C"

namespace moe {
namespace {

// The whole layer; when `ev` is non-NULL, ev[i] is recorded on the stream before stage i
// and ev[MOE_NUM_STAGES] after the last one.
moe_status_t layer_forward_impl(const moe_shape_t* shape, const void* x, const void* centroids,
                                const float* router_bias, const moe_ffn_weights_t* routed, const moe_ffn_weights_t* shared, void* out,
                                int32_t* topk_idx_out, float* topk_gate_out, int32_t* counts_out, void* ws,
                                size_t ws_bytes, cudaStream_t st, cudaEvent_t const* ev, void* ctx = nullptr,
                                size_t ctx_bytes = 0) {
    Dims D;
    MOE_TRY(to_dims(shape, &D));
    if (!centroids || (D.T > 0 && (!x || !out))) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_weights(D, routed, true));
    if (D.Ks > 0) MOE_TRY(check_weights(D, shared));
    else if (shared) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ws(D, ws, ws_bytes));
    if (ctx) {
        MOE_TRY(check_train(D));
        if (ctx_bytes < ctx_layout(D).total || ((uintptr_t)ctx & 15u)) return MOE_ERR_WORKSPACE;
    }
    if (D.T == 0) return MOE_OK;
    MOE_TRY(check_device());
    cudaGetLastError();
    const Layout L = layout(D);
    uint32_t* err = at<uint32_t>(ws, L.err);
    int32_t* idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.idx);
    float* gate = topk_gate_out ? topk_gate_out : at<float>(ws, L.gate);
    int32_t* counts = counts_out ? counts_out : at<int32_t>(ws, L.counts);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* stok = at<int32_t>(ws, L.stok);
    float* sgate = at<float>(ws, L.sgate);
    int32_t* slot_of = at<int32_t>(ws, L.slot_of);
    SavedAG save = {nullptr, nullptr, nullptr, nullptr};
    if (ctx) {          // forward for training: routing, grouping and pre-activations go to ctx
        const CtxLayout C = ctx_layout(D);
        idx = at<int32_t>(ctx, C.idx); gate = at<float>(ctx, C.gate); counts = at<int32_t>(ctx, C.counts);
        offsets = at<int32_t>(ctx, C.offsets); stok = at<int32_t>(ctx, C.stok); sgate = at<float>(ctx, C.sgate);
        slot_of = at<int32_t>(ctx, C.slot_of);
        save = {at<void>(ctx, C.a), at<void>(ctx, C.g), at<void>(ctx, C.as), at<void>(ctx, C.gs)};
    }
    void* y = at<void>(ws, L.y);
    void* hr = at<void>(ws, L.hr);
    void* hs = at<void>(ws, L.hs);
    int32_t* ts1 = at<int32_t>(ws, L.ts1);
    int32_t* ts2 = at<int32_t>(ws, L.ts2);
    const FfnWeights R = to_ffn(routed), Sh = to_ffn(shared);
    auto mark = [&](int i) -> bool { return !ev || cudaEventRecord(ev[i], st) == cudaSuccess; };

    if (!mark(0)) return MOE_ERR_CUDA;
    MOE_TRY(do_route(D, x, centroids, router_bias, idx, gate, at<float>(ws, L.rpart), err, st));
    if (!mark(1)) return MOE_ERR_CUDA;
    MOE_CUDA(launch_permute(D, idx, gate, counts, offsets, stok, sgate, slot_of, at<int32_t>(ws, L.hist), err, st));
    if (!mark(2)) return MOE_ERR_CUDA;
    MOE_CUDA(launch_plan(D, offsets, ts1, ts2, err, st));
    if (!mark(3)) return MOE_ERR_CUDA;
    if (D.q8) {
        uint8_t* x8 = at<uint8_t>(ws, L.xperm);
        float* xs = D.mx ? nullptr : at<float>(ws, L.xs);
        MOE_TRY(quant_gather_x(D, L, ws, x, stok, offsets, ts1, err, st, slot_of));
        if (!mark(4)) return MOE_ERR_CUDA;
        const MxAct m1 = mx_gemm1(L, ws), m2 = mx_gemm2(L, ws);
        MOE_CUDA(launch_tc_gemm1_q8(D, x, x8, xs, offsets, ts1, R, Sh, hr, hs, D.E + D.Ks, err, st,
                                    D.mx ? &m1 : nullptr));
        if (!mark(5)) return MOE_ERR_CUDA;
        uint8_t* h8 = at<uint8_t>(ws, L.h8);
        float* hsc = D.mx ? nullptr : at<float>(ws, L.hsc);
        if (!D.mx)   // block-scaled: GEMM1 already wrote the hidden rows as codes with their run scales
            MOE_CUDA(launch_quant_rows(hr, nullptr, D.slots(), (int)D.slots(), D.I, h8, hsc, err, st));
        float* sout = D.Ks > 0 ? at<float>(ws, L.sout) : nullptr;
        MOE_CUDA(launch_tc_gemm2_routed_q8(D, offsets, ts2, sgate, R, h8, hsc, y, D.Ks > 0 ? &Sh : nullptr, hs, sout,
                                           err, st, D.mx ? &m2 : nullptr));
        if (!mark(6)) return MOE_ERR_CUDA;
        MOE_CUDA(launch_combine(D, y, slot_of, sout, out, err, st));
    } else if (D.bf16) {
        void* xp = at<void>(ws, L.xperm);
        MOE_CUDA(launch_scatter_rows(D, x, slot_of, xp, err, st));     // token order: each row of x read once
        if (!mark(4)) return MOE_ERR_CUDA;
        MOE_CUDA(launch_tc_gemm1(D, x, xp, offsets, ts1, R, Sh, hr, hs, 0, D.E + D.Ks, err, st, ctx ? &save : nullptr));
        if (!mark(5)) return MOE_ERR_CUDA;
        float* sout = D.Ks > 0 ? at<float>(ws, L.sout) : nullptr;
        MOE_CUDA(launch_tc_gemm2_routed(D, offsets, ts2, sgate, R, hr, y, D.Ks > 0 ? &Sh : nullptr, hs, sout, err, st));
        if (!mark(6)) return MOE_ERR_CUDA;
        MOE_CUDA(launch_combine(D, y, slot_of, sout, out, err, st));
    } else {
        if (!mark(4)) return MOE_ERR_CUDA;
        MOE_CUDA(launch_simt_gemm1(D, x, offsets, stok, R, Sh, hr, hs, 0, D.E + D.Ks, err, st));
        if (!mark(5)) return MOE_ERR_CUDA;
        MOE_CUDA(launch_simt_gemm2_routed(D, offsets, sgate, R, hr, y, err, st));
        if (!mark(6)) return MOE_ERR_CUDA;
        if (D.Ks > 0) MOE_CUDA(launch_simt_gemm2_shared(D, Sh, hs, y, slot_of, out, err, st));
        else MOE_CUDA(launch_combine(D, y, slot_of, nullptr, out, err, st));
    }
    if (!mark(7)) return MOE_ERR_CUDA;
    return MOE_OK;
}

// Backward of the layer (moe_layer_backward).
moe_status_t layer_backward_impl(const moe_shape_t* shape, const void* x, const void* centroids,
                                 const float* router_bias, const moe_ffn_weights_t* routed,
                                 const moe_ffn_weights_t* shared, const void* dout, const void* ctx, size_t ctx_bytes,
                                 void* dx, float* dcentroids, float* drouter_bias, const moe_ffn_grads_t* groutes,
                                 const moe_ffn_grads_t* gshared, void* ws, size_t ws_bytes, cudaStream_t st,
                                 cudaEvent_t const* ev = nullptr) {
    Dims D;
    MOE_TRY(to_dims(shape, &D));
    MOE_TRY(check_train(D));
    if (!centroids || !ctx || !dcentroids || (D.T > 0 && (!x || !dout || !dx))) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_weights(D, routed));
    if (D.Ks > 0) MOE_TRY(check_weights(D, shared));
    else if (shared || gshared) return MOE_ERR_INVALID_ARG;
    auto a16 = [](const void* q) { return ((uintptr_t)q & 15u) == 0; };   // 16-byte vector / TMA stores
    auto check_grads = [&](const moe_ffn_grads_t* g) -> bool {
        if (!g || !g->w1 || !g->w3 || !g->w2) return false;
        if (!a16(g->w1) || !a16(g->w3) || !a16(g->w2) || !a16(g->b1) || !a16(g->b3) || !a16(g->b2)) return false;
        const bool b = g->b1 && g->b3 && g->b2, none = !g->b1 && !g->b3 && !g->b2;
        return D.bias ? b : none;
    };
    if (!a16(dx) || !a16(dcentroids)) return MOE_ERR_INVALID_ARG;
    if (!check_grads(groutes) || (D.Ks > 0 && !check_grads(gshared))) return MOE_ERR_INVALID_ARG;
    if (drouter_bias && (!router_bias || D.gate_mode == MOE_GATE_SIGMOID_BIAS)) return MOE_ERR_INVALID_ARG;
    const CtxLayout C = ctx_layout(D);
    if (ctx_bytes < C.total || ((uintptr_t)ctx & 15u)) return MOE_ERR_WORKSPACE;
    const BwdLayout L = bwd_layout(D);
    if (!ws || ws_bytes < L.total || ((uintptr_t)ws & 15u)) return MOE_ERR_WORKSPACE;
    if (D.T == 0) return MOE_OK;
    MOE_TRY(check_device());
    cudaGetLastError();
    uint32_t* err = at<uint32_t>(ws, L.err);
    auto cp = [&](size_t off) { return const_cast<char*>(static_cast<const char*>(ctx)) + off; };
    const int32_t* idx = reinterpret_cast<const int32_t*>(cp(C.idx));
    const int32_t* offsets = reinterpret_cast<const int32_t*>(cp(C.offsets));
    const int32_t* stok = reinterpret_cast<const int32_t*>(cp(C.stok));
    const float* sgate = reinterpret_cast<const float*>(cp(C.sgate));
    const int32_t* slot_of = reinterpret_cast<const int32_t*>(cp(C.slot_of));
    const FfnWeights R = to_ffn(routed), Sh = to_ffn(shared);
    BwdBufs B;
    B.offsets = offsets;
    B.offs_pad = at<int32_t>(ws, L.offs_pad);
    B.ts_dh = at<int32_t>(ws, L.ts_dh);
    B.ts_dx = at<int32_t>(ws, L.ts_dx);
    B.sorted_gate = sgate;
    B.S_pad = L.S_pad_max;
    B.a_sv = cp(C.a); B.g_sv = cp(C.g); B.as_sv = cp(C.as); B.gs_sv = cp(C.gs);
    B.dout_pad = at<void>(ws, L.dout_pad); B.x_pad = at<void>(ws, L.x_pad);
    B.dag = at<void>(ws, L.dag); B.hg = at<void>(ws, L.hg);
    B.dag_s = at<void>(ws, L.dag_s); B.hg_s = at<void>(ws, L.hg_s);
    B.dgate_part = at<float>(ws, L.dgate_part);
    B.dx_slot = at<void>(ws, L.dx_slot);
    B.dz_bf16 = at<void>(ws, L.dz_bf16);
    B.base = at<float>(ws, L.base);
    float* gate_pad = at<float>(ws, L.gate_pad);
    float* b2dot = D.bias ? at<float>(ws, L.b2dot) : nullptr;
    float* z = at<float>(ws, L.z);
    float* dz = at<float>(ws, L.dz);

    auto mark = [&](int i) -> bool { return !ev || cudaEventRecord(ev[i], st) == cudaSuccess; };
    if (!mark(0)) return MOE_ERR_CUDA;
    MOE_CUDA(launch_plan_bwd(D, offsets, const_cast<int32_t*>(B.offs_pad), const_cast<int32_t*>(B.ts_dh),
                             const_cast<int32_t*>(B.ts_dx), st));
    MOE_CUDA(launch_bwd_gather(D, dout, x, R.b2, offsets, B.offs_pad, stok, sgate, B.dout_pad, B.x_pad, B.hg, gate_pad,
                               b2dot, err, st));
    if (D.Ks > 0) MOE_CUDA(launch_fill_aug(B.hg_s, (long long)D.Ks * D.T, D.Is + 64, D.Is, st));
    MOE_CUDA(launch_router_logits(D, x, centroids, z, err, st));
    if (!mark(1)) return MOE_ERR_CUDA;
    MOE_CUDA(launch_tc_dh(D, B, R, Sh, dout, err, st));
    if (!mark(2)) return MOE_ERR_CUDA;
    MOE_CUDA(launch_router_bwd(D, z, router_bias, idx, slot_of, B.dgate_part, L.n_parts, b2dot, dz, B.dz_bf16, nullptr,
                               st));
    if (!mark(3)) return MOE_ERR_CUDA;
    MOE_CUDA(launch_tc_dx(D, B, R, err, st));
    MOE_CUDA(launch_tc_dxs(D, B, Sh, centroids, err, st));
    MOE_CUDA(launch_combine(D, B.dx_slot, slot_of, B.base, dx, err, st));
    if (!mark(4)) return MOE_ERR_CUDA;
    // weight gradients; the routed experts' and the shared experts' w2 bias gradients come out of
    // the same GEMMs through the extra B column (gate, resp. 1)
    const long long T = D.T;
    void* nb = nullptr;
    DwSpec w2 = {0, D.E, D.d, D.I, B.dout_pad, L.S_pad_max, 0, B.hg, L.S_pad_max, 0, B.offs_pad, 0,
                 groutes->w2, nullptr, nullptr, D.I + 64, D.bias ? groutes->b2 : nb, nullptr};
    MOE_CUDA(launch_tc_dw(D, w2, err, st));
    if (!mark(5)) return MOE_ERR_CUDA;
    DwSpec w13 = {1, D.E, 2 * D.I, D.d, B.dag, L.S_pad_max, 0, B.x_pad, L.S_pad_max, 0, B.offs_pad, 0,
                  groutes->w1, groutes->w3, nullptr, D.d + 64, D.bias ? groutes->b1 : nb, D.bias ? groutes->b3 : nb};
    MOE_CUDA(launch_tc_dw(D, w13, err, st));
    if (!mark(6)) return MOE_ERR_CUDA;
    float* cpart = at<float>(ws, L.cpart);
    if (D.Ks > 0) {
        DwSpec s2 = {0, D.Ks, D.d, D.Is, dout, T, 0, B.hg_s, T, 1, nullptr, D.T, gshared->w2, nullptr, nullptr,
                     D.Is + 64, D.bias ? gshared->b2 : nb, nullptr};
        MOE_CUDA(launch_tc_dw(D, s2, err, st));
        DwSpec s13 = {1, D.Ks, 2 * D.Is, D.d, B.dag_s, T, 1, x, T, 0, nullptr, D.T, gshared->w1, gshared->w3, nullptr,
                      0, nullptr, nullptr};
        MOE_CUDA(launch_tc_dw(D, s13, err, st));
        if (D.bias)
            MOE_CUDA(launch_colsum(false, false, B.dag_s, (long long)D.T * 2 * D.Is, 2 * D.Is, D.T, D.Ks, 2 * D.Is, D.Is,
                                   gshared->b1, gshared->b3, cpart, st));
    }
    DwSpec dc = {2, 1, D.E, D.d, B.dz_bf16, T, 0, x, T, 0, nullptr, D.T, nullptr, nullptr, dcentroids, 0, nullptr,
                 nullptr};
    MOE_CUDA(launch_tc_dw(D, dc, err, st));
    if (drouter_bias)
        MOE_CUDA(launch_colsum(true, true, dz, 0, D.E, D.T, 1, D.E, D.E, drouter_bias, nullptr, cpart, st));
    if (!mark(7)) return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" {

MOE_EXPORT moe_status_t moe_layer_forward(const moe_shape_t* shape, const void* x, const void* centroids,
                                          const float* router_bias, const moe_ffn_weights_t* routed, const moe_ffn_weights_t* shared, void* out,
                                          int32_t* topk_idx_out, float* topk_gate_out, int32_t* counts_out, void* ws,
                                          size_t ws_bytes, moe_stream_t stream) {
    return layer_forward_impl(shape, x, centroids, router_bias, routed, shared, out, topk_idx_out, topk_gate_out,
                              counts_out, ws, ws_bytes, (cudaStream_t)stream, nullptr);
}

MOE_EXPORT moe_status_t moe_layer_forward_timed(const moe_shape_t* shape, const void* x, const void* centroids,
                                                const float* router_bias, const moe_ffn_weights_t* routed, const moe_ffn_weights_t* shared,
                                                void* out, int32_t* topk_idx_out, float* topk_gate_out,
                                                int32_t* counts_out, void* ws, size_t ws_bytes, moe_stream_t stream,
                                                void* const* stage_events, int32_t n_events) {
    if (!stage_events || n_events != MOE_NUM_STAGES + 1) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n_events; ++i)
        if (!stage_events[i]) return MOE_ERR_INVALID_ARG;
    return layer_forward_impl(shape, x, centroids, router_bias, routed, shared, out, topk_idx_out, topk_gate_out,
                              counts_out, ws, ws_bytes, (cudaStream_t)stream,
                              reinterpret_cast<cudaEvent_t const*>(stage_events));
}

MOE_EXPORT size_t moe_train_ctx_bytes(const moe_shape_t* shape) {
    Dims D;
    if (to_dims(shape, &D) != MOE_OK || check_train(D) != MOE_OK) return 0;
    return ctx_layout(D).total;
}

MOE_EXPORT size_t moe_backward_workspace_bytes(const moe_shape_t* shape) {
    Dims D;
    if (to_dims(shape, &D) != MOE_OK || check_train(D) != MOE_OK) return 0;
    return bwd_layout(D).total;
}

MOE_EXPORT moe_status_t moe_layer_forward_train(const moe_shape_t* shape, const void* x, const void* centroids,
                                                const float* router_bias, const moe_ffn_weights_t* routed,
                                                const moe_ffn_weights_t* shared, void* out, void* ctx, size_t ctx_bytes,
                                                void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (!ctx) return MOE_ERR_INVALID_ARG;
    return layer_forward_impl(shape, x, centroids, router_bias, routed, shared, out, nullptr, nullptr, nullptr, ws,
                              ws_bytes, (cudaStream_t)stream, nullptr, ctx, ctx_bytes);
}

MOE_EXPORT moe_status_t moe_layer_backward(const moe_shape_t* shape, const void* x, const void* centroids,
                                           const float* router_bias, const moe_ffn_weights_t* routed,
                                           const moe_ffn_weights_t* shared, const void* dout, const void* ctx,
                                           size_t ctx_bytes, void* dx, float* dcentroids, float* drouter_bias,
                                           const moe_ffn_grads_t* routed_grads, const moe_ffn_grads_t* shared_grads,
                                           void* ws, size_t ws_bytes, moe_stream_t stream) {
    return layer_backward_impl(shape, x, centroids, router_bias, routed, shared, dout, ctx, ctx_bytes, dx, dcentroids,
                               drouter_bias, routed_grads, shared_grads, ws, ws_bytes, (cudaStream_t)stream);
}

MOE_EXPORT moe_status_t moe_layer_backward_timed(const moe_shape_t* shape, const void* x, const void* centroids,
                                                 const float* router_bias, const moe_ffn_weights_t* routed,
                                                 const moe_ffn_weights_t* shared, const void* dout, const void* ctx,
                                                 size_t ctx_bytes, void* dx, float* dcentroids, float* drouter_bias,
                                                 const moe_ffn_grads_t* routed_grads,
                                                 const moe_ffn_grads_t* shared_grads, void* ws, size_t ws_bytes,
                                                 moe_stream_t stream, void* const* stage_events, int32_t n_events) {
    if (!stage_events || n_events != MOE_BWD_STAGES + 1) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n_events; ++i)
        if (!stage_events[i]) return MOE_ERR_INVALID_ARG;
    return layer_backward_impl(shape, x, centroids, router_bias, routed, shared, dout, ctx, ctx_bytes, dx, dcentroids,
                               drouter_bias, routed_grads, shared_grads, ws, ws_bytes, (cudaStream_t)stream,
                               reinterpret_cast<cudaEvent_t const*>(stage_events));
}

MOE_EXPORT int32_t moe_backward_launches(const moe_shape_t* shape) {
    Dims D;
    if (to_dims(shape, &D) != MOE_OK || check_train(D) != MOE_OK) return -1;
    if (D.T == 0) return 0;
    int n = 3 + 1 + 1 + 3 + 2 + 1;            // plan, gather, logits; DH; router bwd; DX, DXS, combine; dW2, dW13; dC
    if (D.Ks > 0) n += 3;                      // hg_s bias column, shared dW2, dW13
    if (D.bias && D.Ks > 0) n += 2;            // shared db1 | db3 column sums (two passes)
    return n;                                  // (+2 when a router-bias gradient is asked for)
}

MOE_EXPORT size_t moe_balance_workspace_bytes(const moe_shape_t* shape) {
    Dims D;
    if (to_dims(shape, &D) != MOE_OK || !D.bf16 || !tc_router_supported(D)) return 0;
    return 256 + al((size_t)D.T * D.E * 4) + al((size_t)D.E * ((D.T + 255) / 256) * 4) + al((size_t)D.E * 4);
}

MOE_EXPORT moe_status_t moe_balance_stats(const moe_shape_t* shape, const void* x, const void* centroids,
                                          const float* router_bias, const int32_t* counts, int32_t n_groups, float* f,
                                          float* P, float* terms, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Dims D;
    MOE_TRY(to_dims(shape, &D));
    if (!D.bf16 || !tc_router_supported(D)) return MOE_ERR_UNSUPPORTED;
    if (!x || !centroids || !counts || !f || !P || !terms) return MOE_ERR_INVALID_ARG;
    if (n_groups < 1 || D.E % n_groups || D.E > 1024) return MOE_ERR_INVALID_ARG;
    const size_t need = moe_balance_workspace_bytes(shape);
    if (!ws || ws_bytes < need || ((uintptr_t)ws & 15u)) return MOE_ERR_WORKSPACE;
    if (D.T == 0) return MOE_OK;
    MOE_TRY(check_device());
    cudaGetLastError();
    cudaStream_t st = (cudaStream_t)stream;
    size_t o = 256;
    float* z = at<float>(ws, o); o += al((size_t)D.T * D.E * 4);
    float* partial = at<float>(ws, o); o += al((size_t)D.E * ((D.T + 255) / 256) * 4);
    float* psum = at<float>(ws, o);
    MOE_CUDA(launch_router_logits(D, x, centroids, z, at<uint32_t>(ws, 0), st));
    MOE_CUDA(launch_balance(D, z, router_bias, counts, n_groups, partial, psum, f, P, terms, st));
    return MOE_OK;
}

MOE_EXPORT moe_status_t moe_gather_rows(const void* src, const int32_t* row_of, int64_t n_rows, int64_t src_rows,
                                        int32_t row_bytes, void* dst, void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (n_rows < 0 || src_rows < 0 || row_bytes < 1) return MOE_ERR_INVALID_ARG;
    if (row_bytes % 4) return MOE_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < 256 || ((uintptr_t)ws & 15u)) return MOE_ERR_WORKSPACE;
    if (n_rows == 0) return MOE_OK;
    if (!src || !row_of || !dst) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_device());
    cudaGetLastError();
    MOE_CUDA(launch_gather_rows_generic(src, row_of, n_rows, src_rows, row_bytes, dst, static_cast<uint32_t*>(ws),
                                        (cudaStream_t)stream));
    return MOE_OK;
}

MOE_EXPORT moe_status_t moe_selftest_wait_timeout(uint64_t limit_ns, uint64_t* out, void* ws, size_t ws_bytes,
                                                  moe_stream_t stream) {
    if (limit_ns < 1000ull || limit_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
    if (!ws || ws_bytes < 256 || ((uintptr_t)ws & 15u)) return MOE_ERR_WORKSPACE;
    if (out && ((uintptr_t)out & 7u)) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_device());
    cudaGetLastError();
    MOE_CUDA(launch_wait_selftest(limit_ns, static_cast<uint32_t*>(ws), reinterpret_cast<unsigned long long*>(out),
                                  (cudaStream_t)stream));
    return MOE_OK;
}

MOE_EXPORT moe_status_t moe_segment_ids(const int32_t* counts, int32_t n_segments, int32_t modulo, int64_t n_rows,
                                        int32_t* ids, void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (n_segments < 1 || modulo < 1 || n_rows < 0) return MOE_ERR_INVALID_ARG;
    if (n_segments > SEGMENT_MAX) return MOE_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < 256 || ((uintptr_t)ws & 15u)) return MOE_ERR_WORKSPACE;
    if (n_rows == 0) return MOE_OK;
    if (!counts || !ids) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_device());
    cudaGetLastError();
    MOE_CUDA(launch_segment_ids(counts, n_segments, modulo, n_rows, ids, static_cast<uint32_t*>(ws),
                                (cudaStream_t)stream));
    return MOE_OK;
}

}  // extern "C"
