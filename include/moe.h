/*
 * moe.h — C ABI of the B200 (sm_100a) DeepSeekMoE layer forward.
 *
 * The layer (as defined in "《DeepSeekMoE》深度解读报告", §2.2-§2.3 and §3.1, Eq. 3-5 and
 * Eq. 9-11 in prose, with the per-expert FFN of the `Expert` module in "DeepSeek MoE模型
 * 优化与未来演进及字节超稀疏内存技术"):
 *
 *   z[t,i]   = x[t,:] . centroids[i,:]                      (no scale, no router bias)
 *   s[t,:]   = softmax_i z[t,:]                             (over all N_m routed experts)
 *   picks    = the top_k largest s[t,i]; gate = s at the picks, NOT renormalised
 *   FFN_e(u) = w2_e( silu(w1_e u + b1_e) * (w3_e u + b3_e) ) + b2_e
 *   out[t,:] = sum_{k<K_s} FFN^shared_k(x[t]) + sum_{j<top_k} gate[t,j] * FFN_{idx[t,j]}(x[t])
 *
 * The gate multiplies the whole expert output, bias included.  The residual connection of
 * the original paper is not part of this layer; callers add it.  Ties between equal scores
 * go to the lower expert index; the picks of a token are stored by descending score.
 *
 * Conventions shared by every entry point:
 *  - Every pointer argument is DEVICE memory owned by the caller.  The library allocates
 *    nothing and keeps no state between calls: every intermediate lives in the caller's
 *    workspace `ws` of at least moe_workspace_bytes(shape) bytes (16-byte aligned or better;
 *    256-byte alignment recommended).  One workspace serves every entry point of one shape.
 *  - Every compute call is asynchronous on `stream` (NULL = the legacy default stream) and
 *    does no host synchronisation.  Calls that share a workspace must be ordered on one
 *    stream; calls with distinct workspaces may run concurrently.
 *  - Argument errors are returned synchronously before any launch (MOE_ERR_INVALID_ARG,
 *    MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE).  A failed launch returns MOE_ERR_CUDA.
 *    Errors the kernels detect (an expert index out of range, a bounded wait that ran out)
 *    are recorded in an error word inside the workspace and reported by
 *    moe_check_device_error().  No C++ exception crosses this interface.
 *  - Data types are uniform per call: x, centroids, all weights and biases, hidden states,
 *    routed outputs and `out` share shape->dtype (MOE_F32 or MOE_BF16).  Gates are always
 *    fp32; indices and counts are int32.  Accumulation is fp32 for both data types.
 *  - Layouts are row-major.  Stacked expert weights use the nn.Linear [out, in] layout:
 *    w1, w3: [E, inter, d]; w2: [E, d, inter]; b1, b3: [E, inter]; b2: [E, d].  Bias
 *    pointers must be NULL when has_bias == 0 and non-NULL otherwise.
 *  - Sizes: 0 <= T, T * top_k < 2^31; 1 <= n_experts <= 1024; 1 <= top_k <= min(32,
 *    n_experts); 0 <= n_shared <= 16; d, inter, inter_shared >= 1.  For MOE_BF16, d, inter
 *    and inter_shared must be multiples of 8 (16-byte rows for the tensor-memory-access
 *    unit).  T == 0 is a valid no-op: nothing is launched (moe_permute still writes zero counts
 *    and offsets), and pointers to per-token arrays (x, out, picks, gates, slot lists, routed
 *    rows, dout, dx) may then be NULL, as empty framework tensors' data pointers are.
 *  - FP8 routed experts (shape->routed_fmt == MOE_FMT_E4M3; dtype must be MOE_BF16, d and inter
 *    multiples of 16): the routed w1, w3, w2 are e4m3 codes (1 byte each, same layouts) with
 *    fp32 scales per output channel in s1 [E, inter], s3 [E, inter], s2 [E, d]; the weight is
 *    code * scale.  Each routed expert's input row and each SwiGLU hidden row (rounded to bf16)
 *    is quantised to e4m3 with scale = row max |.| / 448 (division in IEEE fp32, round to
 *    nearest even, saturating), and the expert GEMMs run on the e4m3 tensor-core path with the
 *    scales applied to the fp32 accumulators.  Biases, the router, the shared experts (bf16)
 *    and every output keep shape->dtype.  The pages name FP8 for fine-grained MoE and for
 *    DeepSeek-V3 ("DeepSeek MoE模型优化与未来演进及字节超稀疏内存技术" and the report's §6.2)
 *    without a recipe; this recipe is the library's own.
 *  - Block-scaled FP8 routed experts (shape->routed_fmt == MOE_FMT_MXFP8; same shape rules as
 *    MOE_FMT_E4M3): w1, w3, w2 hold e4m3 codes as above, but each weight row carries one
 *    power-of-two scale per run of 32 consecutive inputs instead of one per row: the scale of a
 *    run is 2^e with e the smallest integer such that max|run| <= 448 * 2^e (0 for an all-zero
 *    run, within [-127, 127]), stored as the byte e + 127 in sf13 (w1 and w3) and sf2 (w2), in
 *    the tiled order moe_quantize_weights_mx writes.  The routed experts' input rows and their
 *    SwiGLU hidden rows (rounded to bf16) are quantised the same way, one such scale per run of
 *    32 along the row.  The tensor cores apply both operands' scales inside the MMA
 *    (kind::mxf8f6f4 with block scales), and the up-projection writes the hidden rows directly
 *    as codes with their scales.  The DeepSeek-V2 explainer (§5.5) advises per-channel or per-group scales
 *    for quantised routed experts, with the shared experts left in 16-bit, as here; it fixes
 *    no group size or scale type.  Groups of 32 with power-of-two scales are what the sm_100a
 *    tensor cores apply natively.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, size out of range, bias pointer mismatch */
    MOE_ERR_UNSUPPORTED = 2, /* valid layer, but outside what these kernels handle */
    MOE_ERR_WORKSPACE = 3,   /* ws NULL or ws_bytes < moe_workspace_bytes(shape) */
    MOE_ERR_CUDA = 4,        /* a CUDA runtime call or a kernel launch failed */
    MOE_ERR_INTERNAL = 5     /* a kernel flagged an error (see moe_check_device_error) */
} moe_status_t;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;

/* Router gate (z = x . e_i + bias_i, bias optional):
 *   MOE_GATE_SOFTMAX_TOPK  softmax of z over all experts, keep it at the top_k largest z,
 *                          no renormalisation ("《DeepSeekMoE》深度解读报告" §3.1; the default).
 *   MOE_GATE_TOPK_SOFTMAX  top_k largest z, softmax over those k logits (gates sum to 1; the
 *                          FineGrainedMoE listing of the DeepSeek-V2 explainer, §3.1, whose
 *                          router is a Linear layer with a bias).
 *   MOE_GATE_SIGMOID_BIAS  s = sigmoid(x . e_i); picks = top_k largest s_i + bias_i (the bias
 *                          steers only the choice); gates = s at the picks over their sum (a
 *                          reading of the sigmoid gate with aux-loss-free balancing the report
 *                          mentions for DeepSeek-V3, §6.2; no formula on the pages). */
typedef enum { MOE_GATE_SOFTMAX_TOPK = 0, MOE_GATE_TOPK_SOFTMAX = 1, MOE_GATE_SIGMOID_BIAS = 2 } moe_gate_mode_t;

/* Storage of the routed experts' weight matrices: MOE_FMT_NATIVE = shape->dtype,
 * MOE_FMT_E4M3 = e4m3 codes with per-output-channel fp32 scales, MOE_FMT_MXFP8 = e4m3 codes
 * with a power-of-two scale per run of 32 inputs (see above). */
typedef enum { MOE_FMT_NATIVE = 0, MOE_FMT_E4M3 = 1, MOE_FMT_MXFP8 = 2 } moe_expert_fmt_t;

typedef struct {
    int32_t T;            /* tokens */
    int32_t d;            /* hidden size */
    int32_t n_experts;    /* N_m, routed experts */
    int32_t inter;        /* intermediate size of a routed expert */
    int32_t top_k;        /* N_r, routed experts per token */
    int32_t n_shared;     /* K_s, shared experts (0 allowed) */
    int32_t inter_shared; /* intermediate size of a shared expert (ignored when n_shared == 0) */
    int32_t has_bias;     /* 1: every Linear has a bias (the page's Expert); 0: no biases */
    int32_t dtype;        /* moe_dtype_t */
    int32_t gate_mode;    /* moe_gate_mode_t (0 = the report's softmax gate) */
    int32_t routed_fmt;   /* moe_expert_fmt_t (0 = weights in dtype) */
} moe_shape_t;

/* One stack of experts (routed: E = n_experts; shared: E = n_shared), nn.Linear layout.
 * Layout hint: when w3 lies a positive multiple of 16 bytes after w1 (for instance the two halves
 * of one [2, E, I, d] buffer), the up-projection fetches a tile's W1 and W3 rows with one request;
 * any other placement is accepted and costs one extra request per pipeline stage. */
typedef struct {
    const void* w1; /* [E, I, d] */
    const void* b1; /* [E, I] or NULL */
    const void* w3; /* [E, I, d] */
    const void* b3; /* [E, I] or NULL */
    const void* w2; /* [E, d, I] */
    const void* b2; /* [E, d] or NULL */
    const float* s1; /* MOE_FMT_E4M3 routed experts: [E, I] scales of w1's rows; NULL otherwise */
    const float* s3; /* MOE_FMT_E4M3: [E, I] scales of w3's rows; NULL otherwise */
    const float* s2; /* MOE_FMT_E4M3: [E, d] scales of w2's rows; NULL otherwise */
    const uint8_t* sf13; /* MOE_FMT_MXFP8 routed experts: scale bytes of w1 and w3 (moe_quantize_weights_mx,
                            MOE_MX_UP, moe_mx_scale_bytes bytes); NULL otherwise */
    const uint8_t* sf2;  /* MOE_FMT_MXFP8: scale bytes of w2 (MOE_MX_DOWN); NULL otherwise */
} moe_ffn_weights_t;

/* Bytes of workspace every entry point needs for this shape (0 if the shape is invalid). */
size_t moe_workspace_bytes(const moe_shape_t* shape);

/* Static description of a status code; never NULL. */
const char* moe_status_string(moe_status_t status);

/* Number of kernel launches one moe_layer_forward call makes for this shape (-1 if the
 * shape is invalid, 0 when T == 0). */
int32_t moe_layer_launches(const moe_shape_t* shape);

/* Library version string, e.g. "moe_b200 0.1 sm_100a". */
const char* moe_version(void);

/* Synchronises `stream`, then reads and clears the error word the kernels keep in `ws`.
 * Returns MOE_OK if no kernel flagged an error since the last check or moe_ws_init(),
 * MOE_ERR_INTERNAL otherwise (*detail, when non-NULL, receives the raw error bits:
 * 1 = expert index out of range, 2 = bounded wait timed out in a GEMM pipeline,
 * 4 = token or slot index out of range).  The only call that synchronises. */
moe_status_t moe_check_device_error(void* ws, size_t ws_bytes, moe_stream_t stream, uint32_t* detail);

/* Clears the workspace's error word (asynchronously on `stream`).  Call once after
 * allocating a workspace; moe_check_device_error() also clears it. */
moe_status_t moe_ws_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Router: scores, top_k picks and gates ("《DeepSeekMoE》深度解读报告" §3.1, Eq. 3-5 in prose,
 * with the variants of shape->gate_mode).
 *   x:           [T, d]           dtype
 *   centroids:   [n_experts, d]   dtype (the expert centroids e_i)
 *   router_bias: [n_experts] fp32 or NULL (no bias)
 *   topk_idx:    [T, top_k] int32 out: expert indices, descending selection key, ties to the
 *                lower index
 *   topk_gate:   [T, top_k] fp32  out: the gate of each pick (see moe_gate_mode_t)
 */
moe_status_t moe_route(const moe_shape_t* shape, const void* x, const void* centroids, const float* router_bias,
                       int32_t* topk_idx, float* topk_gate,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Per-expert token lists (the "top-k indices, then gather tokens per expert" step of the
 * DeepSeek-V2 explainer, eliteato.com/news/32734, §3.1 and §3.3).  Slot s = t*top_k + j.
 * Slots are grouped by expert; inside an expert they keep ascending slot order, so the
 * result is deterministic.
 *   topk_idx, topk_gate: [T, top_k] as produced by moe_route (any values in [0, n_experts))
 *   counts:       [n_experts]     out: slots per expert
 *   offsets:      [n_experts + 1] out: exclusive prefix sum of counts (offsets[E] = T*top_k)
 *   sorted_token: [T*top_k]       out: token of the p-th grouped slot
 *   sorted_gate:  [T*top_k] fp32  out: gate of the p-th grouped slot
 *   slot_of:      [T*top_k]       out: slot_of[s] = grouped position p of slot s
 * An index outside [0, n_experts) sets error bit 1 and the slot is dropped.
 */
moe_status_t moe_permute(const moe_shape_t* shape, const int32_t* topk_idx, const float* topk_gate,
                         int32_t* counts, int32_t* offsets, int32_t* sorted_token,
                         float* sorted_gate, int32_t* slot_of,
                         void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Routed experts on their token lists (the `Expert` module applied per expert):
 *   y_sorted[p, :] = gate_p * FFN_e(x[sorted_token[p], :]) for every grouped position p of
 *   expert e, i.e. offsets[e] <= p < offsets[e+1].  sorted_gate == NULL means gate 1.
 *   x: [T, d]; offsets: [n_experts+1]; sorted_token, sorted_gate: [T*top_k];
 *   routed: stacked weights of the n_experts routed experts; y_sorted: [T*top_k, d] out.
 * offsets must be non-decreasing with offsets[0] = 0 and offsets[E] = T*top_k (as written by
 * moe_permute); sorted_token entries must lie in [0, T) (bit 4 otherwise).
 */
moe_status_t moe_expert_ffn(const moe_shape_t* shape, const void* x, const int32_t* offsets,
                            const int32_t* sorted_token, const float* sorted_gate,
                            const moe_ffn_weights_t* routed, void* y_sorted,
                            void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Shared experts and the combine ("《DeepSeekMoE》深度解读报告" §2.3 and §3.1: the shared
 * experts are summed first, for every token and without the router, then the gated routed
 * outputs are added):
 *   out[t, :] = sum_{k<K_s} FFN^shared_k(x[t]) + sum_{j<top_k} y_sorted[slot_of[t*top_k + j], :]
 * The routed terms are added in ascending j, in fp32, and the sum is rounded once.
 *   x: [T, d]; shared: stacked weights of the K_s shared experts (NULL iff n_shared == 0);
 *   y_sorted: [T*top_k, d]; slot_of: [T*top_k]; out: [T, d] out.
 */
moe_status_t moe_combine(const moe_shape_t* shape, const void* x, const moe_ffn_weights_t* shared,
                         const void* y_sorted, const int32_t* slot_of, void* out,
                         void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The whole layer: moe_route -> moe_permute -> moe_expert_ffn -> moe_combine, all on
 * `stream`, every intermediate in `ws`.
 *   x: [T, d]; centroids: [n_experts, d]; router_bias: [n_experts] fp32 or NULL; routed / shared
 *   weights as above (shared NULL iff n_shared == 0); out: [T, d].
 *   topk_idx_out [T, top_k], topk_gate_out [T, top_k] and counts_out [n_experts] are
 *   optional (NULL = not returned).
 */
moe_status_t moe_layer_forward(const moe_shape_t* shape, const void* x, const void* centroids,
                               const float* router_bias, const moe_ffn_weights_t* routed, const moe_ffn_weights_t* shared,
                               void* out, int32_t* topk_idx_out, float* topk_gate_out,
                               int32_t* counts_out, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_layer_forward with stage timing: identical work and results, and in addition
 * stage_events[i] (each a cudaEvent_t / CUevent created by the caller) is recorded on
 * `stream` before stage i and stage_events[MOE_NUM_STAGES] after the last stage, so that
 * cudaEventElapsedTime between neighbours gives each stage's device time.  Stages, in order:
 *   0 router (scores, softmax, top-k)      1 grouping (histogram, scan, scatter)
 *   2 tile tables of the grouped GEMMs     3 row gather of the routed tokens (bf16 only)
 *   4 GEMM1 + SwiGLU (routed and shared)   5 GEMM2: routed with gates, then (bf16) the
 *                                            shared experts' tiles in the same launch;
 *     (with MOE_FMT_E4M3, stage 3 also quantises the gathered rows and stage 5 starts with
 *      the quantisation of the hidden rows)
 *   6 combine (fp32 layers: shared GEMM2 and combine in one kernel)
 * n_events must be MOE_NUM_STAGES + 1; MOE_ERR_INVALID_ARG otherwise.
 */
#define MOE_NUM_STAGES 7
moe_status_t moe_layer_forward_timed(const moe_shape_t* shape, const void* x, const void* centroids,
                                     const float* router_bias, const moe_ffn_weights_t* routed, const moe_ffn_weights_t* shared,
                                     void* out, int32_t* topk_idx_out, float* topk_gate_out,
                                     int32_t* counts_out, void* ws, size_t ws_bytes, moe_stream_t stream,
                                     void* const* stage_events, int32_t n_events);

/*
 * Per-row e4m3 quantisation of bf16 rows, the step that prepares the FP8 routed experts'
 * inputs (MOE_FMT_E4M3 above), also usable on its own (e.g. for weights: one row = one output
 * channel).  For p in [0, n_rows): r = row_of ? row_of[p] : p;
 *   scale[p]  = max_j |src[r, j]| / 448 (IEEE fp32 division; 1 for an all-zero row)
 *   dst[p, j] = e4m3 code of src[r, j] / scale[p] (IEEE fp32 division, round to nearest even,
 *               saturating at +-448)
 *   src: [src_rows, width] bf16; row_of: [n_rows] int32 or NULL (then n_rows <= src_rows);
 *   dst: [n_rows, width] uint8 out; scale: [n_rows] fp32 out; width a multiple of 8.
 * ws (>= 256 bytes, as for the other calls) only holds the error word: a row_of entry outside
 * [0, src_rows) sets bit 4 and that row comes out as zeros with scale 1.
 */
moe_status_t moe_quantize_rows_e4m3(const void* src, const int32_t* row_of, int64_t n_rows, int32_t src_rows,
                                    int32_t width, uint8_t* dst, float* scale, void* ws, size_t ws_bytes,
                                    moe_stream_t stream);

/*
 * Block-scaled FP8 weights (MOE_FMT_MXFP8): converts a stack of bf16 weight matrices, once,
 * into e4m3 codes and the tiled scale bytes the layer reads.
 *   MOE_MX_UP:   w_a = w1, w_b = w3, each [E, rows = inter, K = d] bf16; codes_a / codes_b
 *                [E, inter, d] uint8 out (for one request per pipeline stage, the two halves of one
 *                [2, E, inter, d] buffer); sf out, shared by w1 and w3.
 *   MOE_MX_DOWN: w_a = w2 [E, rows = d, K = inter] bf16, w_b and codes_b NULL; codes_a [E, d, inter].
 * For every row and every run j of 32 inputs (the last run of a row may be shorter):
 *   e = the smallest integer with max|run| <= 448 * 2^e (0 for an all-zero run), within [-127, 127]
 *   code = e4m3 of value * 2^-e (exact product, round to nearest even)
 * sf (moe_mx_scale_bytes(kind, E, rows, K) bytes, 16-byte aligned) holds the byte e + 127 of
 * each run, tiled as the GEMM stages load it: for rows in groups of P (128 for MOE_MX_UP, 256
 * for MOE_MX_DOWN) and runs in chunks of 4, the 1 KB block ((e * ceil(rows / P) + r / P) *
 * ceil(K / 128) + j / 4) holds two 512-byte halves (MOE_MX_UP: w1, then w3; MOE_MX_DOWN: rows
 * r / 128 even, then odd), and row r's byte for run j sits at (r % 32) * 16 + (r / 32 % 4) * 4
 * + j % 4 of its half; bytes of rows or runs past the matrix are 127.  K must be a multiple of
 * 16 (MOE_ERR_UNSUPPORTED otherwise) and every pointer 16-byte aligned.  Asynchronous on the
 * stream; nothing is allocated and nothing can fail on the device.  No passage on the pages
 * fixes this format (see MOE_FMT_MXFP8 above).
 */
typedef enum { MOE_MX_UP = 0, MOE_MX_DOWN = 1 } moe_mx_kind_t;
size_t moe_mx_scale_bytes(int32_t kind, int32_t n_experts, int32_t rows, int32_t K);
moe_status_t moe_quantize_weights_mx(int32_t kind, const void* w_a, const void* w_b, int32_t n_experts, int32_t rows,
                                     int32_t K, uint8_t* codes_a, uint8_t* codes_b, uint8_t* sf,
                                     moe_stream_t stream);

/*
 * Training: the forward that keeps what the backward needs, and the backward.
 *
 * The pages discuss the backward only through SonicMoE's kernels (the dH kernel, activation
 * memory that does not grow with expert granularity: "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE");
 * the gradients here are the chain rule of the forward above.  Supported layers: MOE_BF16 with
 * native routed weights, a tensor-core router (n_experts a multiple of 16, 16..256) and d, inter,
 * inter_shared multiples of 64; other shapes give MOE_ERR_UNSUPPORTED.
 *
 * The training context (`ctx`, moe_train_ctx_bytes(shape) bytes, caller-owned, 16-byte aligned)
 * holds the picks, gates, grouping and the pre-activations a = x W1^T + b1, g = x W3^T + b3 of
 * every routed slot and shared expert (bf16; T*N_r*inter*4 + K_s*T*inter_shared*4 bytes) and
 * nothing that grows with d*N_r: the expert outputs are not kept.  moe_layer_forward_train writes
 * it (and out, exactly as moe_layer_forward); moe_layer_backward reads it.  Between the two the
 * caller must not change x, the weights or ctx.
 */
typedef struct {
    void* w1; /* [E, I, d], layer dtype */
    void* b1; /* [E, I] or NULL (NULL iff has_bias == 0) */
    void* w3; /* [E, I, d] */
    void* b3; /* [E, I] or NULL */
    void* w2; /* [E, d, I] */
    void* b2; /* [E, d] or NULL */
} moe_ffn_grads_t;

/* Bytes of the training context / of the backward workspace for this shape (0 if the shape
 * is invalid or not supported for training). */
size_t moe_train_ctx_bytes(const moe_shape_t* shape);
size_t moe_backward_workspace_bytes(const moe_shape_t* shape);

/* moe_layer_forward, and in addition the training context in ctx.  ws as for moe_layer_forward. */
moe_status_t moe_layer_forward_train(const moe_shape_t* shape, const void* x, const void* centroids,
                                     const float* router_bias, const moe_ffn_weights_t* routed,
                                     const moe_ffn_weights_t* shared, void* out, void* ctx, size_t ctx_bytes,
                                     void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Gradients of L = <out, dout> for the layer run by moe_layer_forward_train with the same
 * arguments and ctx (the picks are held fixed; they carry no gradient):
 *   dout [T, d] (layer dtype)  in
 *   dx [T, d] (layer dtype)    out: through the routed experts, the shared experts and the router
 *   dcentroids [N_m, d] fp32   out
 *   drouter_bias [N_m] fp32    out, or NULL; must be NULL without a router bias and in gate mode
 *                              MOE_GATE_SIGMOID_BIAS (there the bias only selects)
 *   routed_grads, shared_grads out: weight and bias gradients in the layer dtype (all experts;
 *                              an expert without tokens gets zeros); shared_grads NULL iff
 *                              n_shared == 0
 * dx, dcentroids and every gradient buffer must be 16-byte aligned (MOE_ERR_INVALID_ARG
 * otherwise): they are written with 16-byte vector stores and, for the zeros of experts without
 * tokens, with tensor-memory-access stores.
 * Sums are fp32 on the tensor cores and in fixed order (deterministic); dx adds the routed terms
 * in pick order to the shared and router terms.  ws: moe_backward_workspace_bytes(shape) bytes
 * (its first 256 bytes are the error word, as for the other calls).
 */
moe_status_t moe_layer_backward(const moe_shape_t* shape, const void* x, const void* centroids,
                                const float* router_bias, const moe_ffn_weights_t* routed,
                                const moe_ffn_weights_t* shared, const void* dout, const void* ctx, size_t ctx_bytes,
                                void* dx, float* dcentroids, float* drouter_bias,
                                const moe_ffn_grads_t* routed_grads, const moe_ffn_grads_t* shared_grads,
                                void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_layer_backward with stage timing (as moe_layer_forward_timed): stage_events[i] is recorded
 * before stage i and stage_events[MOE_BWD_STAGES] after the last.  Stages:
 *   0 tile tables, row gathers, router logits    1 dH GEMM (+ SwiGLU backward, gate-gradient partials)
 *   2 router backward (dz)                        3 dx: routed GEMM, shared + router GEMM, combine
 *   4 routed dW2 GEMM                             5 routed dW1 | dW3 GEMM
 *   6 shared experts' dW, dcentroids GEMM, bias-gradient sums
 */
#define MOE_BWD_STAGES 7
moe_status_t moe_layer_backward_timed(const moe_shape_t* shape, const void* x, const void* centroids,
                                      const float* router_bias, const moe_ffn_weights_t* routed,
                                      const moe_ffn_weights_t* shared, const void* dout, const void* ctx,
                                      size_t ctx_bytes, void* dx, float* dcentroids, float* drouter_bias,
                                      const moe_ffn_grads_t* routed_grads, const moe_ffn_grads_t* shared_grads,
                                      void* ws, size_t ws_bytes, moe_stream_t stream, void* const* stage_events,
                                      int32_t n_events);

/* Kernel launches of one moe_layer_backward call without a router-bias gradient (two more with
 * it); -1 for an unsupported shape, 0 when T == 0. */
int32_t moe_backward_launches(const moe_shape_t* shape);

/*
 * Balance statistics of one batch, the quantities the expert- and device-level balance losses of
 * the DeepSeekMoE report are built from (§2.5 and §3: per expert, the batch mean of its gate
 * scores and its hit rate; the formulas are stripped from the page, so these are a reading):
 *   f[i] = N_m / (N_r T) * counts[i]          (1 for every expert under uniform routing)
 *   P[i] = mean over tokens of the score distribution s_t: softmax of the (biased) router logits
 *          over all experts (gate modes 0, 1), or the sigmoid scores normalised over the experts
 *          (mode 2)
 *   terms[0] = sum_i f[i] P[i]                (expert level; a loss multiplies it by alpha1)
 *   terms[1] = sum_g mean_{i in g} f[i] * sum_{i in g} P[i] over n_groups equal contiguous groups
 *              of experts (device level; alpha2)
 * counts [n_experts] int32 as moe_layer_forward's counts_out; f, P [n_experts], terms [2] fp32
 * out.  Needs a bf16 layer with a tensor-core router (it recomputes the logits); fixed
 * summation order (deterministic).  ws: moe_balance_workspace_bytes(shape) bytes.
 */
size_t moe_balance_workspace_bytes(const moe_shape_t* shape);
moe_status_t moe_balance_stats(const moe_shape_t* shape, const void* x, const void* centroids,
                               const float* router_bias, const int32_t* counts, int32_t n_groups, float* f, float* P,
                               float* terms, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Row gather: dst[p, :] = src[row_of[p], :] for p < n_rows, rows of row_bytes bytes (a multiple
 * of 4; 16-byte vectors when row_bytes % 16 == 0 and both buffers are 16-byte aligned).  The
 * expert-parallel layer (the "all_to_all to the experts' devices, then back" scheme of the
 * DeepSeek-V2 explainer, eliteato.com/news/32734, §3.3) moves token rows, gates and expert outputs
 * with it between its exchanges.  A row_of entry outside [0, src_rows) sets error bit 4 in ws
 * (>= 256 bytes) and gives a zero row.
 */
moe_status_t moe_gather_rows(const void* src, const int32_t* row_of, int64_t n_rows, int64_t src_rows,
                             int32_t row_bytes, void* dst, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Self-test of the bounded waits (no counterpart on the pages: a check of this library's hang
 * safety).  Every wait of the tensor-core pipelines is bounded; when one gives up, the kernel
 * sets error bit 2 in ws, stops issuing work, frees its tensor memory and returns, so the
 * context stays usable and moe_check_device_error() reports MOE_ERR_INTERNAL.  This call runs
 * that path on purpose: one warp allocates tensor memory, waits through the same bounded wait
 * on an mbarrier that nothing completes, gives up after limit_ns nanoseconds (1 us .. 10 s),
 * frees the memory and returns.  out (device, 8-byte aligned, may be NULL) receives 2 uint64:
 * 1 if the wait gave up (0 if it completed), and the nanoseconds it waited.  Asynchronous on
 * stream; ws >= 256 bytes (its error word).
 */
moe_status_t moe_selftest_wait_timeout(uint64_t limit_ns, uint64_t* out, void* ws, size_t ws_bytes,
                                       moe_stream_t stream);

/*
 * Segment ids: ids[r] = q mod modulo, where segment q holds row r and the segments are
 * consecutive runs of counts[q] rows (q < n_segments <= 4096), for r < n_rows.  The expert-
 * parallel layer (the all_to_all scheme of the DeepSeek-V2 explainer, eliteato.com/news/32734,
 * §3.3) receives its rows source by source and, inside a source, expert by expert; with
 * counts = the [sources x local experts] received counts and modulo = the local expert count,
 * ids is each received row's local expert, which moe_permute (T = n_rows, top_k = 1) then
 * turns into the expert-major regrouping on the device.  A negative count is taken as 0 and a
 * row past the last segment gets -1; both set error bit 4 in ws (>= 256 bytes).
 * MOE_ERR_UNSUPPORTED for more than 4096 segments.
 */
moe_status_t moe_segment_ids(const int32_t* counts, int32_t n_segments, int32_t modulo, int64_t n_rows,
                             int32_t* ids, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_permute_no_alloc — the paper has no counterpart to this entry point; it exists for
 * callers of this library that cannot allocate device memory.  moe_permute needs scratch
 * space, which it takes from the caller's workspace.  A caller that cannot call cudaMalloc
 * (its framework already gave all device memory to its own caching allocator, it is a
 * plug-in handed only input and output pointers, or it runs on a latency-critical path
 * where an allocation, which may synchronise the device, is not allowed) has no workspace
 * to give.  This variant computes exactly what moe_permute computes (same outputs, bit for
 * bit) but keeps its scratch in a fixed array inside the library, and allocates nothing.
 *
 *   Arguments: as moe_permute, without ws / ws_bytes.  Inputs and outputs are still the
 *   caller's device buffers.
 *   Limit: the scratch is MOE_PERMUTE_NO_ALLOC_SCRATCH_BYTES (1 MiB) per GPU, held by every
 *   GPU that loads the library until the process exits.  A call needs
 *   ceil(T*top_k / 1024) * n_experts * 4 bytes of it (e.g. up to 1,048,576 slots with 256
 *   experts); larger shapes are rejected with MOE_ERR_UNSUPPORTED before any launch.
 *   Set-up: the first call in each CUDA context (a device's primary context, a context the
 *   caller made, or the new primary context after cudaDeviceReset) looks up the scratch's
 *   device address (cudaGetSymbolAddress, with that device current) and keeps it under the
 *   context's process-unique id; make that first call before any stream capture.
 *   Sharing: every call on a device uses the same scratch, which keeps the last call's
 *   contents (nothing in it needs to start at zero).  Calls that overlap on the GPU race:
 *   order them on one stream.
 *   Errors: argument errors as moe_permute (the same shape rules, and MOE_ERR_UNSUPPORTED
 *   on a GPU other than sm_100), checked before any launch.  This variant has no error
 *   word, so unlike every other entry point it does not report bad indices: an expert
 *   index outside [0, n_experts) drops that slot, its slot_of entry is -1 and
 *   offsets[n_experts] comes out smaller than T*top_k.
 */
#define MOE_PERMUTE_NO_ALLOC_SCRATCH_BYTES (1u << 20)
moe_status_t moe_permute_no_alloc(const moe_shape_t* shape, const int32_t* topk_idx, const float* topk_gate,
                                  int32_t* counts, int32_t* offsets, int32_t* sorted_token,
                                  float* sorted_gate, int32_t* slot_of, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
