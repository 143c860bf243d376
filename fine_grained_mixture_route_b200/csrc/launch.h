// Host-side launchers of the sm_100a MoE kernels (internal to the library; the public
// interface is include/moe.h).  Every launcher enqueues on `stream` and returns the
// launch status; none of them synchronises.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Layer sizes in the notation of the DeepSeekMoE report: T tokens, hidden d, E = N_m routed
// experts of intermediate I, k = N_r picks per token, Ks = K_s shared experts of intermediate Is.
struct Dims {
    int T, d, E, I, k, Ks, Is;
    bool bias;
    bool bf16;
    int gate_mode = 0;     // moe_gate_mode_t
    bool q8 = false;       // routed experts in e4m3 (MOE_FMT_E4M3, or MOE_FMT_MXFP8 with mx)
    bool mx = false;       // q8 with block-scaled weights (MOE_FMT_MXFP8)
    long long slots() const { return (long long)T * k; }
};

// ---- router ---------------------------------------------------------------------------
// CUDA-core router for any dtype and N_m <= 1024: block-tiled scores, then one warp per
// token for softmax and top-k.
cudaError_t launch_router_simt(const Dims& D, const void* x, const void* centroids, const float* bias,
                               int32_t* idx, float* gate, cudaStream_t stream);

// ---- per-expert token lists -----------------------------------------------------------
constexpr int PERMUTE_CHUNK = 1024;  // slots per histogram / scatter block
inline int permute_blocks(const Dims& D) { return (int)((D.slots() + PERMUTE_CHUNK - 1) / PERMUTE_CHUNK); }
// Small groupings run the three passes in one block (one launch instead of three).
constexpr long long PERMUTE_SMALL_SLOTS = 16384;
constexpr int PERMUTE_SMALL_EXPERTS = 256;
inline bool permute_small(const Dims& D) {
    return D.slots() > 0 && D.slots() <= PERMUTE_SMALL_SLOTS && D.E <= PERMUTE_SMALL_EXPERTS;
}

cudaError_t launch_permute(const Dims& D, const int32_t* idx, const float* gate, int32_t* counts,
                           int32_t* offsets, int32_t* sorted_token, float* sorted_gate, int32_t* slot_of,
                           int32_t* block_hist, uint32_t* err, cudaStream_t stream);

// Tile tables of the grouped GEMMs.  Groups 0..E-1 are the routed experts (rows from
// offsets, or 0 when offsets is NULL), groups E..E+Ks-1 the shared experts (T rows each).
// tile_start1[G+1]: GEMM1 tiles of GEMM_TILE_ROWS rows x 128 hidden columns; tile_start2[E+1]:
// routed GEMM2 tiles of gemm_tile_rows(D) rows x 256 output columns.
// The expert GEMMs run on CTA pairs (256-row tiles, 128 rows per CTA) when gemm_pairs(D), else
// on single CTAs (128-row tiles).
bool gemm_pairs(const Dims& D);
inline int gemm_tile_rows(const Dims& D) { return gemm_pairs(D) ? 256 : 128; }
cudaError_t launch_plan(const Dims& D, const int32_t* offsets, int32_t* tile_start1, int32_t* tile_start2,
                        uint32_t* err, cudaStream_t stream);

// x_perm[p, :] = x[sorted_token[p], :] (bf16 rows, 16-byte vectors).
cudaError_t launch_gather(const Dims& D, const void* x, const int32_t* sorted_token, void* x_perm,
                          uint32_t* err, cudaStream_t stream);

// The same rows written in token order: x_perm[slot_of[t*k + j], :] = x[t, :] (each row of x
// read once); dropped slots (slot_of -1) are skipped.
cudaError_t launch_scatter_rows(const Dims& D, const void* x, const int32_t* slot_of, void* x_perm, uint32_t* err,
                                cudaStream_t stream);

// Per-row e4m3 quantisation of bf16 rows: for each output row p, src row r = row_of[p] (or p
// when row_of is NULL, r checked against src_rows), scale[p] = max|src[r]| / 448 (1 for a zero
// row), dst[p, :] = e4m3 round-to-nearest-even (saturating) of src[r, :] / scale[p], the
// division in IEEE fp32.  width % 8 == 0.
// Block-scaled e4m3 weights (MOE_FMT_MXFP8): kind 0 = W1 / W3 ([E][rows = I][K = d]; which = 0 for W1,
// 1 for W3; both share one scale array), kind 1 = W2 ([E][rows = d][K = I]).  codes [E][rows][K];
// sf in the tiled order the GEMM stages load (mx_scale_bytes bytes, pre-filled with 127 by the caller).
size_t mx_scale_bytes(int kind, long long n_experts, int rows, int K);
cudaError_t launch_quant_weights_mx(int kind, const void* w, int which, int n_experts, int rows, int K, uint8_t* codes,
                                    uint8_t* sf, cudaStream_t stream);
// Block-scaled routed activations: x rows [rows][K] -> codes [rows][K] and run scales [rows][ceil(K/32)];
// then each grouped position's scales into the GEMM's tiled A-side layout [M-tile][ceil(K/128)][512]
// (mx_act_scale_bytes bytes for `slots` grouped rows; M-tiles numbered by tile_start1 / ceil(I/128)).
size_t mx_act_scale_bytes(long long slots, int n_experts, int K);
cudaError_t launch_quant_rows_mx(const void* src, int rows, int K, uint8_t* codes, uint8_t* sf, cudaStream_t stream);
cudaError_t launch_scatter_sf_tiled(const uint8_t* xsf, int T, int K, const int32_t* stok, const int32_t* offsets,
                                    const int32_t* tile_start1, int E, long long S, int I, uint8_t* sfa, uint32_t* err,
                                    cudaStream_t stream);
cudaError_t launch_quant_rows(const void* src, const int32_t* row_of, long long n_rows, int src_rows, int width,
                              uint8_t* dst, float* scale, uint32_t* err, cudaStream_t stream);
// dst[p, :] = src[row_of[p], :] for rows of row_bytes (a multiple of 4) bytes; bad index -> bit 4, zeros
cudaError_t launch_gather_rows_generic(const void* src, const int32_t* row_of, long long n_rows, long long src_rows,
                                       int row_bytes, void* dst, uint32_t* err, cudaStream_t stream);
// Self-test of the GEMM pipeline's bounded wait: one warp allocates 32 tensor-memory columns,
// waits on an mbarrier that nothing completes until limit_ns pass (error bit 2), frees them;
// out (optional, 2 x u64): 1 if the wait gave up, and the ns waited
cudaError_t launch_wait_selftest(unsigned long long limit_ns, uint32_t* err, unsigned long long* out,
                                 cudaStream_t stream);
// The same move for any rows of row_bytes bytes (a multiple of 16, at most 32 KB, 16-byte aligned
// buffers) by bulk copies through shared memory; with dscale, dscale[slot_of[t*k + j]] = sscale[t].
// cudaErrorNotSupported when the rows or buffers do not qualify (nothing launched).
cudaError_t launch_scatter_rows_bulk(const void* src, const float* sscale, const int32_t* slot_of, int T, int k,
                                     long long S, uint32_t row_bytes, void* dst, float* dscale, uint32_t* err,
                                     cudaStream_t stream);
// dst[slot_of[t*k + j], :] = src[t, :] and dscale[...] = sscale[t] for the picks of each of T
// rows (each source row read once); dropped slots (-1) skipped, positions >= S flagged (bit 4)
cudaError_t launch_scatter_code_rows(const uint8_t* src, const float* sscale, const int32_t* slot_of, int T, int k,
                                     long long S, int row_bytes, uint8_t* dst, float* dscale, uint32_t* err,
                                     cudaStream_t stream);
// ids[r] = (segment holding row r) % modulo for segments of counts[q] consecutive rows
// (n_seg <= SEGMENT_MAX); rows past the last segment get -1 and bit 4, as do negative counts
constexpr int SEGMENT_MAX = 4096;
cudaError_t launch_segment_ids(const int32_t* counts, int n_seg, int modulo, long long n_rows, int32_t* ids,
                               uint32_t* err, cudaStream_t stream);
// dst[p, :] = src[row_of[p], :] for byte rows of row_bytes (a multiple of 16), and dscale[p] =
// sscale[row_of[p]] when dscale is given; an index outside [0, src_rows) sets bit 4 and gives a
// zero row with scale 1.
cudaError_t launch_gather_code_rows(const uint8_t* src, const float* sscale, const int32_t* row_of, long long n_rows,
                                    int src_rows, int row_bytes, uint8_t* dst, float* dscale, uint32_t* err,
                                    cudaStream_t stream);

// out[t, :] = base[t, :] + sum_j y_sorted[slot_of[t*k + j], :] in fp32, rounded once; base is
// the shared experts' fp32 output [T, d], or NULL when there are none.
cudaError_t launch_combine(const Dims& D, const void* y_sorted, const int32_t* slot_of, const float* base,
                           void* out, uint32_t* err, cudaStream_t stream);

// ---- CUDA-core grouped FFN (fp32 layers) ----------------------------------------------
struct FfnWeights {
    const void *w1, *b1, *w3, *b3, *w2, *b2;
    const float *s1 = nullptr, *s3 = nullptr, *s2 = nullptr;   // e4m3 codes: per-output-channel scales
    const uint8_t *sf13 = nullptr, *sf2 = nullptr;              // block-scaled codes: tiled scale bytes
};

// h rows of groups [g_begin, g_end): routed group e -> h_r[offsets[e] + r], shared group
// E + s -> h_s[s*T + r].
cudaError_t launch_simt_gemm1(const Dims& D, const void* x, const int32_t* offsets, const int32_t* sorted_token,
                              const FfnWeights& routed, const FfnWeights& shared, void* h_r, void* h_s,
                              int g_begin, int g_end, uint32_t* err, cudaStream_t stream);
// y_sorted[p] = gate_p * (h_r[p] w2_e^T + b2_e)
cudaError_t launch_simt_gemm2_routed(const Dims& D, const int32_t* offsets, const float* sorted_gate,
                                     const FfnWeights& routed, const void* h_r, void* y_sorted,
                                     uint32_t* err, cudaStream_t stream);
// out[t] = sum_s (h_s[s, t] w2s_s^T + b2s_s) + sum_j y_sorted[slot_of[t*k+j]]   (Ks >= 1)
cudaError_t launch_simt_gemm2_shared(const Dims& D, const FfnWeights& shared, const void* h_s,
                                     const void* y_sorted, const int32_t* slot_of, void* out,
                                     uint32_t* err, cudaStream_t stream);

// ---- tensor-core (tcgen05 / TMEM / TMA) kernels for bf16 layers -------------------------
// All four run the same persistent warp-specialised pipeline: a TMA producer warp, one MMA
// issuing thread, four epilogue warps reading the fp32 accumulators out of tensor memory.
bool tc_router_supported(const Dims& D);
// Split-K policy of the tensor-core router: with few 128-token tiles (decode-sized T) the K
// range is split over CTAs and each writes fp32 partial logits [nsplit][T][N_m]; a CUDA-core
// kernel sums them in split order and does the softmax / top-k.  Returns 1 for no split.
int router_splits(const Dims& D);
inline size_t router_partial_bytes(const Dims& D) {
    const int n = router_splits(D);
    return n > 1 ? (size_t)n * D.T * D.E * sizeof(float) : 0;
}
cudaError_t launch_tc_router(const Dims& D, const void* x, const void* centroids, const float* bias, int32_t* idx,
                             float* gate, float* partial, uint32_t* err, cudaStream_t stream);
cudaError_t launch_router_finish(const Dims& D, const float* partial, int nsplit, const float* bias, int32_t* idx,
                                 float* gate, cudaStream_t stream);
// GEMM1 + SwiGLU over groups [g_begin, g_end): A rows from x_perm (routed) or x (shared).
// Pre-activations a = x W1^T + b1 and g = x W3^T + b3 stored by GEMM1 for the backward pass
// (bf16): routed [T*N_r][I] in grouped order, shared [K_s][T][I_s].
struct SavedAG {
    void *a, *g, *as, *gs;
};
cudaError_t launch_tc_gemm1(const Dims& D, const void* x, const void* x_perm, const int32_t* offsets,
                            const int32_t* tile_start1, const FfnWeights& routed, const FfnWeights& shared,
                            void* h_r, void* h_s, int g_begin, int g_end, uint32_t* err, cudaStream_t stream,
                            const SavedAG* save = nullptr);
// routed GEMM2 with the gate (and b2) applied in the epilogue -> y_sorted; when shared and
// sout are given, the shared experts' GEMM2 tiles (-> fp32 sout, their b2 added) follow the
// routed tiles in the same launch.
cudaError_t launch_tc_gemm2_routed(const Dims& D, const int32_t* offsets, const int32_t* tile_start2,
                                   const float* sorted_gate, const FfnWeights& routed, const void* h_r,
                                   void* y_sorted, const FfnWeights* shared, const void* h_s, float* sout,
                                   uint32_t* err, cudaStream_t stream);
// shared GEMM2: all K_s experts accumulated along K, plus their b2 -> fp32 sout [T, d]
cudaError_t launch_tc_gemm2_shared(const Dims& D, const FfnWeights& shared, const void* h_s, float* sout,
                                   uint32_t* err, cudaStream_t stream);

int num_sms();

// e4m3 routed experts (D.q8).  GEMM1: routed groups read x8_perm rows (scale per row in xs)
// against the W1 / W3 codes (R.s1, R.s3); shared groups [E, g_end) run bf16 on x in the same
// launch.  GEMM2R: h8 rows (scale per row in hs) against the W2 codes (R.s2); with Sh the
// shared experts' bf16 GEMM2 tiles follow (-> sout).
// Block-scaled routed activations (D.mx): the A rows' tiled scale bytes (GEMM1: x codes, GEMM2: h
// codes), and for GEMM1 where the hidden rows go as e4m3 codes [S][I] with their tiled scale bytes.
// The per-row scales (xs, hs) are then unused.
struct MxAct {
    const uint8_t* sfa = nullptr;
    uint8_t* h8 = nullptr;
    uint8_t* sfh = nullptr;
};
cudaError_t launch_tc_gemm1_q8(const Dims& D, const void* x, const void* x8_perm, const float* xs,
                               const int32_t* offsets, const int32_t* tile_start1, const FfnWeights& R,
                               const FfnWeights& Sh, void* h_r, void* h_s, int g_end, uint32_t* err,
                               cudaStream_t stream, const MxAct* mx = nullptr);
cudaError_t launch_tc_gemm2_routed_q8(const Dims& D, const int32_t* offsets, const int32_t* tile_start2,
                                      const float* sorted_gate, const FfnWeights& R, const void* h8,
                                      const float* hs, void* y_sorted, const FfnWeights* Sh, const void* h_s,
                                      float* sout, uint32_t* err, cudaStream_t stream, const MxAct* mx = nullptr);

// ---- backward ----------------------------------------------------------------------
// Buffers of one backward call.  Routed rows of the weight-gradient operands (dout_pad, x_pad,
// dag, hg) are grouped by expert in 64-row-padded groups starting at offs_pad[e] (pad rows zero).
// x_pad rows are d + 64 long and hg / hg_s rows I + 64 / I_s + 64: the first extra column holds 1
// (x_pad, live rows; hg_s) or the slot's gate (hg), so the weight-gradient GEMMs also produce
// the bias gradients (sum over rows of dag, resp. of gate * dout).
struct BwdBufs {
    const int32_t *offsets, *offs_pad, *ts_dh, *ts_dx;
    const float* sorted_gate;
    long long S_pad;
    const void *a_sv, *g_sv, *as_sv, *gs_sv;     // saved pre-activations (forward for training)
    void *dout_pad, *x_pad;                      // [S_pad][d]
    void *dag, *hg;                              // [S_pad][2I], [S_pad][I]
    void *dag_s, *hg_s;                          // [K_s][T][2I_s], [K_s][T][I_s]
    float* dgate_part;                           // [S][2 * ceil(I / 256)]
    void* dx_slot;                               // [S][d]
    void* dz_bf16;                               // [T][N_m]
    float* base;                                 // [T][d] fp32: shared experts' dx + router dx
};
// One weight-gradient GEMM: per group, out[M][N] = A^T B over the group's rows (K), with A
// [rows][M] and B [rows][N] row-major (MN-major operands).  rows: group row starts [groups+1]
// into 2-D operands, or null with K rows per group (3-D operands index the group, 2-D ones are
// shared by all groups).  kind 0: out0 [groups][M][N]; 1: rows < M/2 -> out0, the rest -> out1
// (each [groups][M/2][N]); 2: out_f32 [groups][M][N].
// With bias0 set, B has a column N (its rows' weights: the gate, or 1) whose output column is a
// bias gradient: out column N -> bias0[g][M] (kind 1: rows < M/2 -> bias0[g][M/2], the rest ->
// bias1); b_ld is B's row length (>= N + 1 then; 0 means N).
struct DwSpec {
    int kind, groups, M, N;
    const void* a; long long a_rows; int a3d;
    const void* b; long long b_rows; int b3d;
    const int32_t* rows; int K;
    void *out0, *out1;
    float* out_f32;
    int b_ld;
    void *bias0, *bias1;
};
cudaError_t launch_router_logits(const Dims& D, const void* x, const void* centroids, float* z, uint32_t* err,
                                 cudaStream_t stream);
cudaError_t launch_tc_dh(const Dims& D, const BwdBufs& B, const FfnWeights& R, const FfnWeights& Sh, const void* dout,
                         uint32_t* err, cudaStream_t stream);
cudaError_t launch_tc_dx(const Dims& D, const BwdBufs& B, const FfnWeights& R, uint32_t* err, cudaStream_t stream);
cudaError_t launch_tc_dxs(const Dims& D, const BwdBufs& B, const FfnWeights& Sh, const void* centroids, uint32_t* err,
                          cudaStream_t stream);
cudaError_t launch_tc_dw(const Dims& D, const DwSpec& w, uint32_t* err, cudaStream_t stream);
// offs_pad[E+1] (64-row-padded group starts), ts_dh[E+Ks+1], ts_dx[E+1] from the grouping offsets
cudaError_t launch_plan_bwd(const Dims& D, const int32_t* offsets, int32_t* offs_pad, int32_t* ts_dh, int32_t* ts_dx,
                            cudaStream_t stream);
// padded grouped rows of dout and x, the padded gate column, and b2dot[p] = <dout_t, b2_e> (b2 may be null)
cudaError_t launch_bwd_gather(const Dims& D, const void* dout, const void* x, const void* b2, const int32_t* offsets,
                              const int32_t* offs_pad, const int32_t* stok, const float* sgate, void* dout_pad,
                              void* x_pad, void* hg, float* gate_pad, float* b2dot, uint32_t* err, cudaStream_t stream);
// gate gradients -> logit gradients dz [T][N_m] (fp32 and bf16); dgate_out [T][k] optional
cudaError_t launch_router_bwd(const Dims& D, const float* z, const float* bias, const int32_t* idx,
                              const int32_t* slot_of, const float* dgate_part, int n_parts, const float* b2dot,
                              float* dz, void* dz_bf16, float* dgate_out, cudaStream_t stream);
// column sums over n_rows rows of each group (two passes through partial [groups][ceil(n_rows/256)][W]
// fp32, deterministic); see backward.cu
cudaError_t launch_colsum(bool src_f32, bool out_f32, const void* src, long long group_stride, int ld, int n_rows,
                          int groups, int W, int split, void* out0, void* out1, float* partial, cudaStream_t stream);
// balance statistics from the router logits z [T][N_m] (turned into scores in place) and the hit
// counts: f, P [N_m], terms [2] (expert-level, device-level over n_groups)
cudaError_t launch_balance(const Dims& D, float* z, const float* bias, const int32_t* counts, int n_groups,
                           float* partial, float* psum, float* f, float* P, float* terms, cudaStream_t stream);
// rows[r][col] = 1 and rows[r][col + 1 .. col + 63] = 0 (bf16), r < n_rows
cudaError_t launch_fill_aug(void* rows, long long n_rows, int ld, int col, cudaStream_t stream);

}  // namespace moe
