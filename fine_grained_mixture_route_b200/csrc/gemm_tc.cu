// Tensor-core kernels of the DeepSeekMoE layer: one persistent, warp-specialised tcgen05
// pipeline whose modes differ in their tile tables, operand loads and epilogues.
//
// Forward:
//   ROUTER  scores z = x C^T of 128 tokens x N_m experts; the epilogue thread that owns a
//           token row does the softmax over all N_m experts and the top-N_r selection
//           ("《DeepSeekMoE》深度解读报告" §3.1, Eq. 3-5 in prose).
//   ROUTERP split-K variant of ROUTER for few token tiles: fp32 partial logits per K range,
//           summed and ranked by a small CUDA-core kernel afterwards.
//   GEMM1   [x_e] [w1_e | w3_e]^T for 128 rows x (128 + 128) columns with bias and SwiGLU in
//           the epilogue: h = silu(x w1^T + b1) * (x w3^T + b3) (the `Expert` module of
//           "DeepSeek MoE模型优化与未来演进及字节超稀疏内存技术").  Routed groups read the
//           expert's gathered rows, shared groups read x itself.
//   GEMM2R  routed w2 contraction; the epilogue adds b2 and scales by the gate: the gate
//           multiplies the whole expert output.
//   GEMM2S  the K_s shared experts' w2 contractions accumulated along K in one accumulator;
//           the epilogue adds the shared biases and writes the fp32 shared output, to which
//           the combine kernel adds each token's gated routed rows in pick order (§2.3 and
//           §3.1 of the DeepSeekMoE report: shared experts first, then the gated routed sum).
//   Q8      GEMM1 / GEMM2R with e4m3 routed tiles (kind::f8f6f4, per-row scales applied to
//           the fp32 accumulator in the epilogue); shared tiles of the same launch stay bf16.
// Backward (MN-major B operands, read through 4-D TMA views, one request per stage):
//   DH      dout W2 with the SwiGLU backward and the gate-gradient partial sums in the epilogue;
//   DX      [da | dg] [W1 ; W3] per routed slot;  DXS  shared experts + dz C per token (fp32);
//   DW      weight gradients, both operands MN-major, K = a group's rows; groups without rows
//           are zero-filled by the producer's TMA stores and skip the MMA and epilogue.
//
// Pipeline (320 threads, one CTA per SM, persistent over a static round-robin tile order):
//   warp 0      TMA producer: 128B-swizzled tiles of A (16 KB) and B (up to 32 KB) into a
//               4-stage shared-memory ring, completion counted on mbarriers;
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma (M=128, N<=256,
//               bf16 K=16 or e4m3 K=32, fp32 accumulate) and commits each stage back to the
//               producer and each finished accumulator to the epilogue;
//   warps 2-9   epilogue: tcgen05.ld of their 32 TMEM lanes (one accumulator row per
//               thread; the two warps of a lane quadrant split the columns), fp32 math,
//               stores through a per-warp shared-memory transpose.  Two accumulators
//               (2 x 256 columns) let the epilogue of one tile overlap the main loop of the next.
// Every mbarrier wait is bounded (a few seconds of %globaltimer); on expiry the kernel sets
// an error bit, stops issuing, waits (bounded) for its own copies and MMAs in flight, frees
// TMEM and returns.  A CTA-pair variant of the expert GEMMs (cta_group::2, clusters of two,
// off by default) is in the source; no TMA load anywhere uses cluster multicast.
#include <cuda.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace tc {
bool pairs_for(const Dims& D);

constexpr int BM = 128;                  // rows per CTA (TMEM lanes)
constexpr int BK = 64;                   // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int A_BYTES = BM * BK * 2;     // 16 KB
constexpr int THREADS = 320;              // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int EPI_WARPS = 8;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 256;
constexpr int RING_BYTES = 192 * 1024;   // shared-memory ring (stages x (A + B))
constexpr int STAGE_OUT_BYTES = 2048;     // per epilogue warp: a 32 x 32 bf16 chunk being transposed
constexpr int SMEM_BYTES = 1024 /*align slack*/ + RING_BYTES + 256 /*barriers*/ + EPI_WARPS * STAGE_OUT_BYTES;
constexpr int ZERO_BYTES = 16384;         // DW: zeros that TMA stores copy to the gradients of groups without rows
constexpr int SMEM_BYTES_DW = SMEM_BYTES + ZERO_BYTES;
// Block-scaled operands (mxw): each stage also brings the B tile's scale bytes (256 rows x 4
// runs of 32 = 1 KB, two 512-byte blocks of 128 rows each, row r at byte (r % 32) * 16 +
// (r / 32 % 4) * 4 + run) and the A tile's (128 rows, one such 512-byte block), copied from
// there into tensor-memory columns SFB_COL..SFB_COL + 7 and SFA_COL..SFA_COL + 3 before the
// stage's MMAs.  To free those columns the second accumulator starts MX_OVL columns early
// (224 instead of 256), so the two accumulators share columns 224-255: the epilogue drains
// that shared chunk first and releases it through ovl_bar before the next tile's MMAs start.
constexpr int MX_OVL = 32;
constexpr int SF_STAGE_BYTES = 1024;                             // B scales of one stage
constexpr int SFA_BYTES = 512;                                   // A scales of one stage
constexpr uint32_t SFA_COL = 2 * ACC_COLS - MX_OVL;            // 480
constexpr uint32_t SFB_COL = SFA_COL + 8;                        // 488
constexpr int SMEM_BYTES_Q8 = SMEM_BYTES + 4 * (SF_STAGE_BYTES + SFA_BYTES);
constexpr unsigned long long WAIT_NS = 4000000000ull;
#ifndef MOE_GROUP_M
#define MOE_GROUP_M 8                    // M-tiles per raster band of the expert GEMMs
#endif
constexpr uint32_t PEER_BIT_MASK = 0xFEFFFFFFu;   // shared::cluster address of CTA rank 0 of a pair

enum Mode : int { ROUTER = 0, GEMM1 = 1, GEMM2R = 2, GEMM2S = 3, ROUTERP = 4, DH = 5, DX = 6, DXS = 7, DW = 8 };
// Backward modes (B operand MN-major: contraction along rows, 64-column boxes):
//   DH  dh = dout . W2 per routed / shared group, SwiGLU backward and the gate gradient in the epilogue
//   DX  dx per routed slot = [da | dg] . [W1 ; W3]
//   DXS shared experts' dx + the router's dz . C, accumulated along K, fp32 per token
//   DW  weight gradients: A and B both MN-major, K = the rows (tokens) of a group

// The expert GEMMs can run on CTA pairs (cta_group::2): a 256-row tile, each CTA holding 128
// rows of A, half of the 256 B rows and its 128 x 256 slice of the accumulator, so each SM
// loads 32 KB per K stage instead of 48 KB.  Pairs pay off when experts hold many rows; with a
// few rows per expert (decode) single CTAs keep twice as many weight tiles in flight.  The
// router modes always run on single CTAs.
template <int MODE, bool PAIR_ = false>
struct Cfg {
    static constexpr bool PAIR = PAIR_ && (MODE == GEMM1 || MODE == GEMM2R || MODE == GEMM2S);
    static constexpr int TM = PAIR ? 2 * BM : BM;                 // rows per tile
    static constexpr int B_BYTES = (PAIR ? 128 : 256) * BK * 2;   // B rows held by one CTA
    static constexpr int STAGES = RING_BYTES / (A_BYTES + B_BYTES);
};

struct Params {
    CUtensorMap tmA[2];
    CUtensorMap tmB[4];
    CUtensorMap tmZ[2];        // DW (dw_zero): the gradient outputs, 2-D, box dw_zbw x 32 rows, no swizzle
    const int32_t* tile_start;
    const int32_t* offsets;
    int g_begin, g_end;
    int T, d, E, I, Is, k, Ks;
    int n_mma;                 // MMA N (256, or N_m for the router)
    long long S;
    const __nv_bfloat16 *b1, *b3, *b2, *sb1, *sb3, *sb2;
    __nv_bfloat16* h_r;
    __nv_bfloat16* h_s;
    const float* sorted_gate;
    __nv_bfloat16* y;
    float* sout;               // GEMM2S: fp32 shared-expert output [T][d]
    int32_t* idx_out;
    float* gate_out;
    const float* router_bias;  // ROUTER / ROUTERP: optional per-expert bias [E]
    int gate_mode;             // ROUTER: moe_gate_mode_t
    float* partial;            // ROUTERP: [nsplit][T][E] fp32 partial logits
    int kb_per_split;          // ROUTERP: K blocks per split
    int group_m;               // tile raster: bands of group_m M-tiles swept across all N-tiles
    int q8;                    // routed tiles read e4m3 A and B (K blocks of 128 bytes)
    const float* a_scale;      // q8: per-row scale of the routed A rows (x_perm or h rows)
    const float *ws1, *ws3, *ws2;  // q8: per-output-channel weight scales [E, I], [E, I], [E, d]
    int mxw;                   // q8, block-scaled: the MMAs apply the operands' run scales
    const uint8_t* sf13;       // mxw: W1 | W3 scale bytes, [E][ceil(I/128)][ceil(d/128)][W1, W3][512]
    const uint8_t* sf2;        // mxw: W2 scale bytes, [E][ceil(d/256)][ceil(I/128)][2][512]
    const uint8_t* sfa;        // mxw: the routed A rows' scale bytes, [M-tile][K chunk][512]
    uint8_t* h8_out;           // mxw GEMM1: routed hidden rows as e4m3 codes [S][I] ...
    uint8_t* sfh_out;          // ... and their scale bytes, [M-tile][ceil(I/128)][512] (GEMM2's sfa)
    int fold_shared;           // GEMM2R: shared-expert GEMM2 tiles follow the routed ones (-> sout)
    // ---- forward for training: GEMM1 also stores the pre-activations a = x W1^T + b1, g = x W3^T + b3
    __nv_bfloat16 *a_out, *g_out;      // routed [S][I] (grouped order)
    __nv_bfloat16 *as_out, *gs_out;    // shared [Ks][T][Is]
    // ---- backward
    const int32_t* offs_pad;           // [E+1] starts of the 64-row-padded groups (dout / x / dag / hg rows)
    const __nv_bfloat16 *a_sv, *g_sv;  // saved pre-activations, routed [S][I]
    const __nv_bfloat16 *as_sv, *gs_sv;  // shared [Ks][T][Is]
    __nv_bfloat16 *dag, *hg;           // DH out, routed: [S_pad][2I] (da | dg), [S_pad][I] (gate * h)
    __nv_bfloat16 *dag_s, *hg_s;       // DH out, shared: [Ks][T][2Is], [Ks][T][Is]
    float* dgate_part;                 // DH out: [S][n_parts] partial sums of dh_raw * h
    int n_parts;
    __nv_bfloat16* dx_slot;            // DX out: [S][d] (grouped order)
    int dw_kind;                       // DW: 0 out [g][M][N]; 1 rows < M/2 -> out0, rest -> out1; 2 fp32 [M][N]
    int dw_groups, dw_M, dw_N;         // DW: groups and output rows / columns per group
    int dw_a3d, dw_b3d;                // DW: operand map is 3-D (third coordinate = group)
    const int32_t* dw_rows;            // DW: group row starts [groups+1] (padded), or null: rows = dw_K
    int dw_K;
    __nv_bfloat16 *dw_out0, *dw_out1;
    float* dw_out_f32;
    int dw_Nt;                         // DW: columns the tiles cover (dw_N, or dw_N + 1 with a bias column)
    int dw_bias_col;                   // DW: B column dw_N holds the row weights of a bias gradient (or -1):
    __nv_bfloat16 *dw_bias0, *dw_bias1;  //    out column dw_N -> bias0 [g][M] (kind 1: rows >= M/2 -> bias1)
    int dw_zero;                       // DW: a group without rows is written by the producer's TMA stores of
    int dw_zbw;                        //    zeros (box dw_zbw columns x 32 rows); its tiles skip MMA and epilogue
    int w13_one;                       // GEMM1: bit 0 routed, bit 1 shared: tmB[0] / tmB[2] is a 4-D view
                                       // {d, I, W1 | W3, expert} and one request brings both weight blocks
    int mn_wide;                       // MN-major operands read through 4-D views {64 columns, rows, column
                                       // blocks, groups}: one request per operand and stage instead of one per
                                       // 64-column block (DW: tmA[1] / tmB[1]; DH, DX, DXS: their B maps)
    uint32_t* err;
};

// ------------------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait on the phase `parity` of an mbarrier: true once it completes; false when the
// pipeline was aborted (abort_flag set by another role) or the wait gave up after limit_ns of
// %globaltimer or WAIT_MAX_POLLS polls, whichever comes first; giving up sets abort_flag and
// error bit 2.
constexpr uint32_t WAIT_MAX_POLLS = 1u << 30;
__device__ __forceinline__ bool mbar_wait_limit(uint32_t bar, uint32_t parity, volatile int* abort_flag, uint32_t* err,
                                                bool honour_abort, unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0u) {
            if (honour_abort && *abort_flag) return false;
            if (globaltimer() - t0 > limit_ns || i >= WAIT_MAX_POLLS) {
                *abort_flag = 1;
                flag_error(err, ERR_PIPE_TIMEOUT);
                return false;
            }
        }
    }
}
// The pipeline's wait: a few seconds at most.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, uint32_t* err,
                                       bool honour_abort = true) {
    return mbar_wait_limit(bar, parity, abort_flag, err, honour_abort, WAIT_NS);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"((unsigned long long)map), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
            dst),
        "l"((unsigned long long)map), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1, int c2,
                                            int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(
            dst),
        "l"((unsigned long long)map), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)map) : "memory");
}
// shared -> global tensor store (bulk-group completion); the box starts inside the tensor and
// is clipped at its far edges
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     (unsigned long long)map),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
// shared -> global bulk copy of `bytes` (multiple of 16; both addresses 16-byte aligned)
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"((unsigned long long)dst), "r"(src),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row core-matrix
// groups 1024 bytes apart (stride byte offset); leading byte offset unused for this layout;
// descriptor version 1 (bits 46-47); layout type 2 = SWIZZLE_128B (bits 61-63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// Shared-memory descriptor of an MN-major operand, 128-byte swizzle: 64-element rows along MN,
// 8-row K groups 1024 bytes apart (stride byte offset), 64-wide MN blocks 8 KB apart (leading
// byte offset: one TMA box of 64 K rows each).
__device__ __forceinline__ uint64_t mn_sw128_desc(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(8192 >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
constexpr uint32_t IDESC_A_MN = 1u << 15, IDESC_B_MN = 1u << 16;   // operand major-ness bits
// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both K-major, M=128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// Instruction descriptor, kind::f8f6f4: fp32 accumulator, e4m3 A and B (format 0), K-major, M=128.
__host__ __device__ constexpr uint32_t idesc_e4m3(int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
// One e4m3 MMA: K = 32 (32 bytes of each operand row, like the 16 bf16 of mma_bf16).
__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// ---- block-scaled e4m3 weights (moe_expert_fmt_t MOE_FMT_MXFP8)
// Instruction descriptor, kind::mxf8f6f4 with block scales: fp32 accumulator, e4m3 A and B
// (format 0), K-major, M = 128, scale factors UE8M0 (bit 23); the byte of each 32-bit scale
// column that an MMA reads is selected per operand (A: bits 29-30, B: bits 4-5).
__host__ __device__ constexpr uint32_t idesc_mx(int n, int sf_byte) {
    return ((uint32_t)sf_byte << 4) | ((uint32_t)(n >> 3) << 17) | (1u << 23) | ((uint32_t)(BM >> 4) << 24) |
           ((uint32_t)sf_byte << 29);
}
// One block-scaled e4m3 MMA (K = 32): D (+)= (A * 2^sfa[row]) (B * 2^sfb[col])^T, where the scale
// of A row r is the UE8M0 byte sf_byte of tensor-memory lane r, column sfa + r / 32, and the scale
// of B row n likewise from column sfb + n / 32.  The byte index travels in bits 30-31 of the two
// scale addresses as well as in the descriptor.
__device__ __forceinline__ void mma_mx(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
}
// Shared-memory descriptor of a 32-row x 16-byte block (four 8-row core matrices, 128 bytes
// apart), no swizzle: the source of a 32x128b copy into tensor memory.
__device__ __forceinline__ uint64_t sf_desc(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(128 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}
// Copy 32 rows x 128 bits of shared memory into tensor-memory columns taddr .. taddr + 3 of
// lanes 0-31, repeated in the other three lane quarters (asynchronous; ordered before the MMAs
// this thread issues after it).
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) global -> shared,
// completing on the mbarrier's transaction count.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ---- CTA-pair (cta_group::2) forms
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on the pair leader's
// barrier (the peer bit of the barrier address cleared).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            dst),
        "l"((unsigned long long)map), "r"(bar & PEER_BIT_MASK), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                                 int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
            dst),
        "l"((unsigned long long)map), "r"(bar & PEER_BIT_MASK), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// arrive (when this thread's MMAs finish) on the barrier at the same offset in both CTAs
__device__ __forceinline__ void mma_commit_pair_both(uint32_t bar) {
    const uint16_t mask = 0x3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"(mask)
        : "memory");
}
__device__ __forceinline__ void mma_commit_pair_local(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// plain arrive on the barrier at the same offset in CTA rank 0 of the cluster
__device__ __forceinline__ void mbar_arrive_rank0(uint32_t bar) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(remote) : "r"(bar));
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}
// Instruction descriptor for the pair MMA: M = 256 (128 rows per CTA).
// kind::f8f6f4 e4m3 MMA across a CTA pair (M = 256)
__device__ __forceinline__ void mma_e4m3_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__host__ __device__ constexpr uint32_t idesc_e4m3_pair(int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_bf16_pair(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

// ------------------------------------------------------------------------------ tile order
struct Tile {
    int g;       // group: expert (routed), E + s (shared GEMM1), 0 otherwise
    int m0;      // first row of the tile inside its group
    int n0;      // first output column
    int rows;    // rows of the group
    int row0;    // first row of the group in A and in the output
    int num_kb;  // K blocks of 64
    int kb0;     // first K block (split-K router)
};

template <int MODE, bool PAIR>
__device__ __forceinline__ int total_tiles(const Params& p) {
    constexpr int TM = Cfg<MODE, PAIR>::TM;
    if (MODE == ROUTER) return ceil_div(p.T, TM);
    if (MODE == ROUTERP) return ceil_div(p.T, TM) * ceil_div(ceil_div(p.d, BK), p.kb_per_split);
    if (MODE == GEMM1) return p.tile_start[p.g_end] - p.tile_start[p.g_begin];
    if (MODE == GEMM2R)
        return p.tile_start[p.E] + (p.fold_shared ? ceil_div(p.T, TM) * ceil_div(p.d, 256) : 0);
    if (MODE == DH) return p.tile_start[p.E + p.Ks];
    if (MODE == DX) return p.tile_start[p.E];
    if (MODE == DW) return p.dw_groups * ceil_div(p.dw_M, TM) * ceil_div(p.dw_Nt, 256);
    return ceil_div(p.T, TM) * ceil_div(p.d, 256);
}

// largest g in [lo, hi) with ts[g] <= t   (ts non-decreasing, ts[hi] > t)
__device__ __forceinline__ int find_group(const int32_t* ts, int lo, int hi, int t) {
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (ts[mid] <= t) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Banded raster inside a group of mt x nt tiles: bands of up to gm M-tiles; inside a band the
// M-tile index runs fastest, then N.  CTAs working at the same time then share a few A row
// blocks and sweep the B tiles of one band, which keeps both in L2.
__device__ __forceinline__ void band_mn(int local, int mt, int nt, int gm, int& m, int& n) {
    const int band = local / (gm * nt);
    const int rem = local - band * gm * nt;
    const int rows = min(gm, mt - band * gm);
    n = rem / rows;
    m = band * gm + rem % rows;
}

template <int MODE, bool PAIR>
__device__ __forceinline__ Tile decode(const Params& p, int t) {
    constexpr int TM = Cfg<MODE, PAIR>::TM;
    Tile x;
    x.kb0 = 0;
    if (MODE == ROUTER) {
        x.g = 0; x.m0 = t * TM; x.n0 = 0; x.rows = p.T; x.row0 = 0; x.num_kb = ceil_div(p.d, BK);
    } else if (MODE == ROUTERP) {
        const int mt = ceil_div(p.T, TM);
        const int split = t / mt;
        const int kbt = ceil_div(p.d, BK);
        x.g = split; x.m0 = (t % mt) * TM; x.n0 = 0; x.rows = p.T; x.row0 = 0;
        x.kb0 = split * p.kb_per_split;
        x.num_kb = min(p.kb_per_split, kbt - x.kb0);
    } else if (MODE == GEMM1) {
        const int tt = t + p.tile_start[p.g_begin];
        const int g = find_group(p.tile_start, p.g_begin, p.g_end, tt);
        const int local = tt - p.tile_start[g];
        const bool shared = g >= p.E;
        x.g = g;
        x.rows = shared ? p.T : p.offsets[g + 1] - p.offsets[g];
        x.row0 = shared ? 0 : p.offsets[g];
        const int mt = ceil_div(x.rows, TM);
        int m, n;
        band_mn(local, mt, ceil_div(shared ? p.Is : p.I, 128), p.group_m, m, n);
        x.m0 = m * TM;
        x.n0 = n * 128;
        x.num_kb = ceil_div(p.d, (p.q8 && !shared) ? 2 * BK : BK);
    } else if (MODE == DH) {
        const int g = find_group(p.tile_start, 0, p.E + p.Ks, t);
        const int local = t - p.tile_start[g];
        const bool shared = g >= p.E;
        x.g = g;
        x.rows = shared ? p.T : p.offsets[g + 1] - p.offsets[g];
        x.row0 = shared ? 0 : p.offs_pad[g];
        int m, n;
        band_mn(local, ceil_div(x.rows, TM), ceil_div(shared ? p.Is : p.I, 256), p.group_m, m, n);
        x.m0 = m * TM;
        x.n0 = n * 256;
        x.num_kb = ceil_div(p.d, BK);
    } else if (MODE == DX) {
        const int e = find_group(p.tile_start, 0, p.E, t);
        const int local = t - p.tile_start[e];
        x.g = e;
        x.rows = p.offsets[e + 1] - p.offsets[e];
        x.row0 = p.offs_pad[e];
        int m, n;
        band_mn(local, ceil_div(x.rows, TM), ceil_div(p.d, 256), p.group_m, m, n);
        x.m0 = m * TM;
        x.n0 = n * 256;
        x.num_kb = 2 * ceil_div(p.I, BK);
    } else if (MODE == DXS) {
        x.g = 0; x.rows = p.T; x.row0 = 0;
        int m, n;
        band_mn(t, ceil_div(p.T, TM), ceil_div(p.d, 256), p.group_m, m, n);
        x.m0 = m * TM;
        x.n0 = n * 256;
        x.num_kb = p.Ks * 2 * ceil_div(p.Is, BK) + ceil_div(p.E, BK);
    } else if (MODE == DW) {
        const int mt = ceil_div(p.dw_M, TM), nt = ceil_div(p.dw_Nt, 256);
        const int g = t / (mt * nt);
        int m, n;
        band_mn(t - g * mt * nt, mt, nt, p.group_m, m, n);
        x.g = g;
        x.m0 = m * TM;
        x.n0 = n * 256;
        x.row0 = p.dw_rows ? p.dw_rows[g] : 0;
        x.rows = p.dw_rows ? p.dw_rows[g + 1] - p.dw_rows[g] : p.dw_K;
        x.num_kb = ceil_div(x.rows, BK);
    } else if (MODE == GEMM2R && t >= p.tile_start[p.E]) {
        // shared-expert tile (fold_shared): all K_s experts accumulated along K
        const int mt = ceil_div(p.T, TM);
        x.g = -1; x.rows = p.T; x.row0 = 0;
        int m, n;
        band_mn(t - p.tile_start[p.E], mt, ceil_div(p.d, 256), p.group_m, m, n);
        x.m0 = m * TM;
        x.n0 = n * 256;
        x.num_kb = p.Ks * ceil_div(p.Is, BK);
    } else if (MODE == GEMM2R) {
        const int e = find_group(p.tile_start, 0, p.E, t);
        const int local = t - p.tile_start[e];
        x.g = e;
        x.rows = p.offsets[e + 1] - p.offsets[e];
        x.row0 = p.offsets[e];
        const int mt = ceil_div(x.rows, TM);
        int m, n;
        band_mn(local, mt, ceil_div(p.d, 256), p.group_m, m, n);
        x.m0 = m * TM;
        x.n0 = n * 256;
        x.num_kb = ceil_div(p.I, p.q8 ? 2 * BK : BK);
    } else {
        const int mt = ceil_div(p.T, TM);
        x.g = 0; x.rows = p.T; x.row0 = 0;
        int m, n;
        band_mn(t, mt, ceil_div(p.d, 256), p.group_m, m, n);
        x.m0 = m * TM;
        x.n0 = n * 256;
        x.num_kb = p.Ks * ceil_div(p.Is, BK);
    }
    return x;
}

// ------------------------------------------------------------------------------ epilogues
// Top-k insertion keeping (value desc, index asc); candidates arrive in ascending index.
// Top-k insertion keeping (key desc, index asc) with a payload; candidates arrive in ascending
// index, so an equal key never displaces an earlier (lower-index) entry.
template <int KMAX>
__device__ __forceinline__ void topk_insert(float (&tv)[KMAX], int (&ti)[KMAX], float (&tp)[KMAX], float v, int e,
                                            float payload) {
    if (v > tv[KMAX - 1]) {
        tv[KMAX - 1] = v;
        ti[KMAX - 1] = e;
        tp[KMAX - 1] = payload;
#pragma unroll
        for (int j = KMAX - 1; j > 0; --j) {
            if (tv[j] > tv[j - 1]) {
                float a = tv[j]; tv[j] = tv[j - 1]; tv[j - 1] = a;
                int b = ti[j]; ti[j] = ti[j - 1]; ti[j - 1] = b;
                float c = tp[j]; tp[j] = tp[j - 1]; tp[j - 1] = c;
            }
        }
    }
}

// Router epilogue: the thread owning a token row reads its N_m logits from TMEM.  Selection key
// z + bias (gate modes 0, 1) or sigmoid(z) + bias (mode 2); gates: mode 0 the softmax of z + bias
// over all experts at the picks (a second pass sums the exponentials), mode 1 the softmax over
// the k picked keys, mode 2 the picks' sigmoids divided by their sum.
template <int KMAX>
__device__ __forceinline__ void epilogue_router(const Params& p, const Tile& x, uint32_t tacc, int row) {
    float tv[KMAX], tp[KMAX];
    int ti[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) { tv[j] = -INFINITY; ti[j] = 0; tp[j] = 0.f; }
    const int mode = p.gate_mode;
    for (int c0 = 0; c0 < p.n_mma; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(tacc + c0, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int e = c0 + j;
            if (e < p.E) {
                const float z = __uint_as_float(r[j]);
                const float bb = p.router_bias ? p.router_bias[e] : 0.f;
                if (mode == 2) {
                    const float sg = 1.0f / (1.0f + expf(-z));
                    topk_insert<KMAX>(tv, ti, tp, sg + bb, e, sg);
                } else {
                    topk_insert<KMAX>(tv, ti, tp, z + bb, e, z + bb);
                }
            }
        }
    }
    float gsum = 0.f;
    if (mode == 0) {
        const float zmax = tv[0];
        for (int c0 = 0; c0 < p.n_mma; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(tacc + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (c0 + j < p.E)
                    gsum += expf(__uint_as_float(r[j]) + (p.router_bias ? p.router_bias[c0 + j] : 0.f) - zmax);
        }
    }
    const int t = x.m0 + row;
    if (t < p.T) {
        float g[KMAX];
        float norm = 0.f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (mode == 0) g[j] = expf(tp[j] - tv[0]) / gsum;
            else if (mode == 1) g[j] = expf(tp[j] - tp[0]);
            else g[j] = tp[j];
            if (j < p.k) norm += g[j];
        }
        const float rn = mode == 0 ? 1.f : 1.0f / norm;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < p.k) {
                p.idx_out[(size_t)t * p.k + j] = ti[j];
                p.gate_out[(size_t)t * p.k + j] = g[j] * rn;
            }
        }
    }
}

// Stores a warp's 32 x 32 bf16 chunk (lane = row, pk = its 32 columns packed in pairs) through a
// per-warp shared-memory transpose, so that each store instruction writes 64 contiguous bytes of
// eight rows instead of 16 bytes of 32 rows.  In shared memory row r keeps its four 16-byte pieces
// rotated by r/2, which makes both the writes and the reads free of bank conflicts.  row_ptr is
// this lane's destination row (already offset to column 0 of the chunk), or null to skip the row;
// ncols (multiple of 8) limits the columns written.
__device__ __forceinline__ void warp_store_chunk_bf16(uint32_t stage, const uint32_t (&pk)[16], __nv_bfloat16* row_ptr,
                                                      int ncols, int lane) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t a = stage + lane * 64 + (((j + (lane >> 1)) & 3) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * j]), "r"(pk[4 * j + 1]),
                     "r"(pk[4 * j + 2]), "r"(pk[4 * j + 3])
                     : "memory");
    }
    __syncwarp();
    const int j = lane & 3;
#pragma unroll
    for (int sgrp = 0; sgrp < 4; ++sgrp) {
        const int r = sgrp * 8 + (lane >> 2);
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(
            __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(row_ptr), r));
        uint4 v;
        const uint32_t a = stage + r * 64 + (((j + (r >> 1)) & 3) << 4);
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
        if (dst && j * 8 < ncols) *reinterpret_cast<uint4*>(dst + j * 8) = v;
    }
    __syncwarp();
}

// GEMM1: the two epilogue warps of a TMEM lane quadrant split the 128 hidden columns.  On an
// e4m3 routed tile (Q8) the accumulators are first multiplied by the row's activation scale
// and the column's weight scale.  Rows are stored through the per-warp transpose (all lanes
// take part; rows past the group's end pass a null row).
// Block-scaled routed tile (mxw): the global index of its 128-row block among all routed experts'
// blocks (expert e's blocks start at tile_start[e] / N-tiles per block), which indexes the A-side
// scale bytes [M-tile][K chunk][512].  GEMM1 and GEMM2 number the blocks alike.
template <int MODE>
__device__ __forceinline__ int mx_mtile(const Params& p, const Tile& x) {
    const int ntn = MODE == GEMM1 ? ceil_div(p.I, 128) : ceil_div(p.d, 256);
    return p.tile_start[x.g] / ntn + x.m0 / BM;
}

// Block-scaled tiles: offset of the scale byte of tile row r (0-127), run j, in the tiled layout
// [M-tile][K chunk of 128][512] (row r at (r % 32) * 16 + (r / 32 % 4) * 4 + j % 4 of its chunk).
__device__ __forceinline__ size_t mx_scale_byte(int mtile, int chunks, int r, int j) {
    return ((size_t)mtile * chunks + j / 4) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (j & 3);
}

// One run of 32 hidden values (bf16-rounded, packed in pk) of this thread's row -> e4m3 codes
// with the smallest non-saturating power-of-two scale: ncols codes to dst (null for a padding
// row, which stores only the neutral scale byte 127), the exponent byte to *sf.
__device__ __forceinline__ void store_run_e4m3(const Params& p, const uint32_t (&pk)[16], uint8_t* dst, int ncols,
                                               uint8_t* sf) {
    (void)p;
    float v[32];
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        v[2 * i] = __uint_as_float(pk[i] << 16);
        v[2 * i + 1] = __uint_as_float(pk[i] & 0xFFFF0000u);
        if (2 * i < ncols) m = fmaxf(m, fabsf(v[2 * i]));
        if (2 * i + 1 < ncols) m = fmaxf(m, fabsf(v[2 * i + 1]));
    }
    const int ex = dst ? mx_exponent(m) : 0;
    *sf = (uint8_t)(ex + 127);
    if (!dst) return;
    const float mul = __uint_as_float((uint32_t)(127 - ex) << 23);   // 2^-ex (ex <= 126 for finite h)
    uint32_t q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i] * mul, v[4 * i + 1] * mul), __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi =
            __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i + 2] * mul, v[4 * i + 3] * mul), __NV_SATFINITE, __NV_E4M3);
        q[i] = lo | (hi << 16);
    }
    if (ncols == 32) {
        reinterpret_cast<uint4*>(dst)[0] = make_uint4(q[0], q[1], q[2], q[3]);
        reinterpret_cast<uint4*>(dst)[1] = make_uint4(q[4], q[5], q[6], q[7]);
    } else {
        for (int j = 0; j < ncols; ++j) dst[j] = (uint8_t)(q[j >> 2] >> (8 * (j & 3)));
    }
}

// Overlapping accumulators (mxw): the warp that holds the columns both accumulators share
// reports them drained (their tensor-memory loads complete) so the next tile's MMAs may start.
__device__ __forceinline__ void release_shared_cols(uint32_t ovl, int lane) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(ovl);
}

// ovl (mxw): 0, or the barrier this warp releases after loading the shared chunk, which it then
// loads first (ovl_last: the shared chunk is the last of this warp's chunks).
template <bool Q8 = false>
__device__ __forceinline__ void epilogue_gemm1(const Params& p, const Tile& x, uint32_t tacc, int row, int half,
                                               uint32_t stage, int lane, uint32_t ovl = 0, bool ovl_last = false) {
    const bool shared = x.g >= p.E;
    const int e = shared ? x.g - p.E : x.g;
    const int I = shared ? p.Is : p.I;
    const __nv_bfloat16* b1 = shared ? p.sb1 : p.b1;
    const __nv_bfloat16* b3 = shared ? p.sb3 : p.b3;
    if (b1) b1 += (size_t)e * I;
    if (b3) b3 += (size_t)e * I;
    const bool scaled = Q8 && !shared;          // e4m3 routed tile
    const float* sc1 = (scaled && !p.mxw) ? p.ws1 + (size_t)e * I : nullptr;   // block-scaled: in the MMA
    const float* sc3 = (scaled && !p.mxw) ? p.ws3 + (size_t)e * I : nullptr;
    const int r = x.m0 + row;
    const bool live = r < x.rows;
    // block-scaled tiles: the input rows' scales are applied by the MMA, and h leaves as e4m3 codes
    // with one scale per run of 32 (this thread's 32-column chunk) for GEMM2's A operand
    const bool mxq = scaled && p.mxw;
    const float rs = (scaled && !p.mxw && live) ? p.a_scale[x.row0 + r] : 1.f;
    const size_t ro = shared ? ((size_t)e * p.T + r) * I : (size_t)(x.row0 + r) * I;
    const int mtile = mxq ? mx_mtile<GEMM1>(p, x) : 0;
    __nv_bfloat16* hrow = live ? (shared ? p.h_s : p.h_r) + ro : nullptr;
    __nv_bfloat16* arow = (live && p.a_out) ? (shared ? p.as_out : p.a_out) + ro : nullptr;
    __nv_bfloat16* grow = (live && p.a_out) ? (shared ? p.gs_out : p.g_out) + ro : nullptr;
#pragma unroll 1
    for (int it = 0; it < 2; ++it) {
        const int c = half * 2 + (ovl_last ? 1 - it : it);
        uint32_t u[32], v[32];
        tmem_ld32(tacc + c * 32, u);
        tmem_ld32(tacc + 128 + c * 32, v);
        tmem_wait_ld();
        if (ovl && it == 0) release_shared_cols(ovl, lane);
        const int col0 = x.n0 + c * 32;
        if (col0 >= I) {                                        // warp-uniform
            // block-scaled: a run past I inside GEMM2's last K chunk still gets a finite scale
            // byte (its codes are zero there), so no scale that GEMM2 reads is left unset
            if (mxq && col0 / 128 < ceil_div(I, 128))
                p.sfh_out[mx_scale_byte(mtile, ceil_div(I, 128), row, col0 / 32)] = 127;
            continue;
        }
        const int ncols = min(32, I - col0);
        uint32_t pk[16], pa[16], pg[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float hv[2], av[2], gv[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = 2 * i + h;
                const int cc = min(col0 + j, I - 1);
                float a = __uint_as_float(u[j]);
                float g = __uint_as_float(v[j]);
                if (scaled) {
                    a *= rs * (sc1 ? sc1[cc] : 1.f);
                    g *= rs * (sc3 ? sc3[cc] : 1.f);
                }
                a += b1 ? __bfloat162float(b1[cc]) : 0.f;
                g += b3 ? __bfloat162float(b3[cc]) : 0.f;
                hv[h] = silu_f32(a) * g;
                av[h] = a;
                gv[h] = g;
            }
            pk[i] = pack_bf16(hv[0], hv[1]);
            pa[i] = pack_bf16(av[0], av[1]);
            pg[i] = pack_bf16(gv[0], gv[1]);
        }
        if (mxq) {                                              // warp-uniform
            store_run_e4m3(p, pk, live ? p.h8_out + ro + col0 : nullptr, ncols,
                           p.sfh_out + mx_scale_byte(mtile, ceil_div(I, 128), row, col0 / 32));
            continue;
        }
        warp_store_chunk_bf16(stage, pk, hrow ? hrow + col0 : nullptr, ncols, lane);
        if (p.a_out) {                                          // warp-uniform
            warp_store_chunk_bf16(stage, pa, arow ? arow + col0 : nullptr, ncols, lane);
            warp_store_chunk_bf16(stage, pg, grow ? grow + col0 : nullptr, ncols, lane);
        }
    }
}

// GEMM2R: each epilogue warp of a quadrant takes 128 of the 256 output columns.  On e4m3 tiles
// (Q8) the accumulator is multiplied by the h row's scale and the column's weight scale before
// b2 and the gate.  Rows are stored through the per-warp transpose.
template <bool Q8 = false>
__device__ __forceinline__ void epilogue_gemm2r(const Params& p, const Tile& x, uint32_t tacc, int row, int half,
                                                uint32_t stage, int lane, uint32_t ovl = 0, bool ovl_last = false) {
    const int r = x.m0 + row;
    const bool live = r < x.rows;
    const long long pos = x.row0 + r;
    const float gate = live ? (p.sorted_gate ? p.sorted_gate[pos] : 1.f) : 0.f;
    const __nv_bfloat16* b2 = p.b2 ? p.b2 + (size_t)x.g * p.d : nullptr;
    const float* sc2 = (Q8 && !p.mxw) ? p.ws2 + (size_t)x.g * p.d : nullptr;   // block-scaled: in the MMA
    const float rs = (Q8 && !p.mxw && live) ? p.a_scale[pos] : 1.f;
    __nv_bfloat16* yrow = live ? p.y + (size_t)pos * p.d : nullptr;
#pragma unroll 1
    for (int it = 0; it < 4; ++it) {
        const int c = half * 4 + (ovl_last ? (it + 3) % 4 : it);
        uint32_t u[32];
        tmem_ld32(tacc + c * 32, u);
        tmem_wait_ld();
        if (ovl && it == 0) release_shared_cols(ovl, lane);
        const int col0 = x.n0 + c * 32;
        if (col0 >= p.d) continue;                              // warp-uniform
        const int ncols = min(32, p.d - col0);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int ca = min(col0 + 2 * i, p.d - 1), cb = min(col0 + 2 * i + 1, p.d - 1);
            float a = __uint_as_float(u[2 * i]);
            float b = __uint_as_float(u[2 * i + 1]);
            if (Q8) {
                a *= rs * (sc2 ? sc2[ca] : 1.f);
                b *= rs * (sc2 ? sc2[cb] : 1.f);
            }
            a += b2 ? __bfloat162float(b2[ca]) : 0.f;
            b += b2 ? __bfloat162float(b2[cb]) : 0.f;
            pk[i] = pack_bf16(gate * a, gate * b);
        }
        warp_store_chunk_bf16(stage, pk, yrow ? yrow + col0 : nullptr, ncols, lane);
    }
}

// GEMM2S: the shared experts' output (accumulator + their b2 summed), fp32, for the combine.
__device__ __forceinline__ void epilogue_gemm2s(const Params& p, const Tile& x, uint32_t tacc, int row, int half,
                                                uint32_t ovl = 0, int lane = 0, bool ovl_last = false) {
    const int t = x.m0 + row;
    const bool live = t < p.T;
    float* srow = p.sout + (size_t)t * p.d;
#pragma unroll 1
    for (int it = 0; it < 4; ++it) {
        const int c = half * 4 + (ovl_last ? (it + 3) % 4 : it);
        uint32_t u[32];
        tmem_ld32(tacc + c * 32, u);
        tmem_wait_ld();
        if (ovl && it == 0) release_shared_cols(ovl, lane);
        const int col0 = x.n0 + c * 32;
        if (!live || col0 >= p.d) continue;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int col = col0 + q * 4;
            if (col >= p.d) break;
            float4 v = make_float4(__uint_as_float(u[q * 4]), __uint_as_float(u[q * 4 + 1]),
                                   __uint_as_float(u[q * 4 + 2]), __uint_as_float(u[q * 4 + 3]));
            if (p.sb2)
                for (int s = 0; s < p.Ks; ++s) {
                    const __nv_bfloat16* b = p.sb2 + (size_t)s * p.d + col;
                    v.x += __bfloat162float(b[0]); v.y += __bfloat162float(b[1]);
                    v.z += __bfloat162float(b[2]); v.w += __bfloat162float(b[3]);
                }
            *reinterpret_cast<float4*>(srow + col) = v;
        }
    }
}

// ROUTERP (split-K router): each thread writes its token row's partial logits over this
// tile's K range; the two warps of a quadrant alternate 16-column groups.
__device__ __forceinline__ void epilogue_router_partial(const Params& p, const Tile& x, uint32_t tacc, int row,
                                                        int half) {
    const int t = x.m0 + row;
    float* dst = p.partial + ((size_t)x.g * p.T + t) * p.E;
    for (int c0 = half * 16; c0 < p.n_mma; c0 += 32) {
        uint32_t r[16];
        tmem_ld16(tacc + c0, r);
        tmem_wait_ld();
        if (t < p.T) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<float4*>(dst + c0 + q * 4) =
                    make_float4(__uint_as_float(r[q * 4]), __uint_as_float(r[q * 4 + 1]), __uint_as_float(r[q * 4 + 2]),
                                __uint_as_float(r[q * 4 + 3]));
        }
    }
}

// DH: for a routed group the rows are grouped slots (A = dout rows of the slot's token, in the
// 64-row-padded layout), for a shared group the tokens.  Per element of the hidden row:
// dh_raw = (dout . W2)[c]; a, g = the saved pre-activations; sg = sigmoid(a); h = a sg g;
// dh = gate dh_raw; da = dh g sg (1 + a (1 - sg)); dg = dh a sg; and the row's partial sum of
// dh_raw h (the gate gradient, without its b2 term) over this thread's 128 columns.  Writes da | dg
// and gate * h (the B operand of the w2 gradient); the padding rows of a routed group (up to the
// next multiple of 64) get zeros, so the weight-gradient GEMMs can run whole 64-row K blocks.
__device__ __forceinline__ void epilogue_dh(const Params& p, const Tile& x, uint32_t tacc, int row, int half,
                                            uint32_t stage, int lane) {
    const bool shared = x.g >= p.E;
    const int e = shared ? x.g - p.E : x.g;
    const int I = shared ? p.Is : p.I;
    const int r = x.m0 + row;
    const bool live = r < x.rows;
    const bool pad = !shared && !live && r < ceil_div(x.rows, 64) * 64;
    const long long pu = shared ? r : (long long)p.offsets[e] + r;       // grouped slot (routed) / token
    const long long pp = shared ? r : (long long)x.row0 + r;             // padded row (routed) / token
    const size_t so = shared ? ((size_t)e * p.T + r) * I : (size_t)pu * I;
    const __nv_bfloat16* arow = (shared ? p.as_sv : p.a_sv) + so;
    const __nv_bfloat16* grow = (shared ? p.gs_sv : p.g_sv) + so;
    __nv_bfloat16* dagrow = nullptr;
    __nv_bfloat16* hgrow = nullptr;
    if (live || pad) {
        dagrow = shared ? p.dag_s + ((size_t)e * p.T + r) * 2 * I : p.dag + (size_t)pp * 2 * I;
        // gate * h rows carry 64 extra columns (the bias-gradient column of the w2 gradient GEMM)
        hgrow = shared ? p.hg_s + ((size_t)e * p.T + r) * (I + 64) : p.hg + (size_t)pp * (I + 64);
    }
    const float gate = (!shared && live) ? p.sorted_gate[pu] : 1.f;
    float dot = 0.f;
#pragma unroll 1
    for (int c = half * 4; c < half * 4 + 4; ++c) {
        uint32_t u[32];
        tmem_ld32(tacc + c * 32, u);
        tmem_wait_ld();
        const int col0 = x.n0 + c * 32;
        if (col0 >= I) continue;                                // warp-uniform
        uint32_t pda[16], pdg[16], phg[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint4 av = make_uint4(0, 0, 0, 0), gv = make_uint4(0, 0, 0, 0);
            if (live) {
                av = *reinterpret_cast<const uint4*>(arow + col0 + q * 8);
                gv = *reinterpret_cast<const uint4*>(grow + col0 + q * 8);
            }
            const uint32_t aw[4] = {av.x, av.y, av.z, av.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float da2[2], dg2[2], hg2[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float a = __uint_as_float(h ? (aw[i] & 0xFFFF0000u) : (aw[i] << 16));
                    const float g = __uint_as_float(h ? (gw[i] & 0xFFFF0000u) : (gw[i] << 16));
                    const float dhr = live ? __uint_as_float(u[q * 8 + i * 2 + h]) : 0.f;
                    const float sg = 1.0f / (1.0f + expf(-a));
                    const float si = a * sg;
                    const float hv = si * g;
                    dot += dhr * hv;
                    const float dh = gate * dhr;
                    da2[h] = dh * g * sg * (1.0f + a * (1.0f - sg));
                    dg2[h] = dh * si;
                    hg2[h] = gate * hv;
                }
                pda[q * 4 + i] = pack_bf16(da2[0], da2[1]);
                pdg[q * 4 + i] = pack_bf16(dg2[0], dg2[1]);
                phg[q * 4 + i] = pack_bf16(hg2[0], hg2[1]);
            }
        }
        // I is a multiple of 64: whole chunks
        warp_store_chunk_bf16(stage, pda, dagrow ? dagrow + col0 : nullptr, 32, lane);
        warp_store_chunk_bf16(stage, pdg, dagrow ? dagrow + I + col0 : nullptr, 32, lane);
        warp_store_chunk_bf16(stage, phg, hgrow ? hgrow + col0 : nullptr, 32, lane);
    }
    if (!shared && live) p.dgate_part[(size_t)pu * p.n_parts + (x.n0 / 256) * 2 + half] = dot;
}

// DX: dx of a routed slot (grouped order), bf16, stored through the per-warp transpose.
__device__ __forceinline__ void epilogue_dx(const Params& p, const Tile& x, uint32_t tacc, int row, int half,
                                            uint32_t stage, int lane) {
    const int r = x.m0 + row;
    const bool live = r < x.rows;
    __nv_bfloat16* orow = live ? p.dx_slot + ((size_t)p.offsets[x.g] + r) * p.d : nullptr;
#pragma unroll 1
    for (int c = half * 4; c < half * 4 + 4; ++c) {
        uint32_t u[32];
        tmem_ld32(tacc + c * 32, u);
        tmem_wait_ld();
        const int col0 = x.n0 + c * 32;
        if (col0 >= p.d) continue;                              // warp-uniform
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1]));
        warp_store_chunk_bf16(stage, pk, orow ? orow + col0 : nullptr, min(32, p.d - col0), lane);
    }
}

// Second half of warp_store_chunk_bf16 with the eight-row destinations precomputed: dst[sg] is the
// row (sg * 8 + lane / 4) of the warp's 32 rows, already offset to this chunk's column 0.
__device__ __forceinline__ void warp_store_chunk_pre(uint32_t stage, const uint32_t (&pk)[16],
                                                     __nv_bfloat16* const (&dst)[4], int ncols, int lane) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t a = stage + lane * 64 + (((j + (lane >> 1)) & 3) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * j]), "r"(pk[4 * j + 1]),
                     "r"(pk[4 * j + 2]), "r"(pk[4 * j + 3])
                     : "memory");
    }
    __syncwarp();
    const int j = lane & 3;
#pragma unroll
    for (int sgrp = 0; sgrp < 4; ++sgrp) {
        const int r = sgrp * 8 + (lane >> 2);
        uint4 v;
        const uint32_t a = stage + r * 64 + (((j + (r >> 1)) & 3) << 4);
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
        if (dst[sgrp] && j * 8 < ncols) *reinterpret_cast<uint4*>(dst[sgrp] + j * 8) = v;
    }
    __syncwarp();
}

// DW: one 128 x 256 tile of a group's weight gradient (zeros when the group has no rows).  bf16
// outputs go through the per-warp transpose; the four chunks of a warp are loaded from tensor
// memory one ahead of the one being stored.  Column dw_N, when it is the bias column, goes to
// the bias gradient.
__device__ __forceinline__ void dw_chunk(const Params& p, const Tile& x, const uint32_t (&u)[32], int c, int m,
                                         bool live, int Mh, __nv_bfloat16* orow, float* frow,
                                         __nv_bfloat16* const (&drow)[4], uint32_t stage, int lane) {
    const int col0 = x.n0 + c * 32;
    if (col0 >= p.dw_Nt) return;                               // warp-uniform
    const bool zero = x.num_kb == 0;
    if (live && p.dw_bias_col >= 0 && col0 + 32 > p.dw_N && col0 <= p.dw_N) {
        // dw_N is a multiple of 64 (d, inter, inter_shared are) and chunks start at multiples of
        // 32, so the bias column is the chunk's first column
        const __nv_bfloat16 bv = __float2bfloat16_rn(zero ? 0.f : __uint_as_float(u[0]));
        if (p.dw_kind == 1) {
            if (m < Mh) p.dw_bias0[(size_t)x.g * Mh + m] = bv;
            else p.dw_bias1[(size_t)x.g * Mh + m - Mh] = bv;
        } else {
            p.dw_bias0[(size_t)x.g * p.dw_M + m] = bv;
        }
    }
    const int ncols = min(32, p.dw_N - col0);
    if (ncols <= 0) return;                                     // warp-uniform
    if (p.dw_kind == 2) {
        if (!live) return;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (q * 4 < ncols)
                *reinterpret_cast<float4*>(frow + col0 + q * 4) =
                    zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                         : make_float4(__uint_as_float(u[q * 4]), __uint_as_float(u[q * 4 + 1]),
                                       __uint_as_float(u[q * 4 + 2]), __uint_as_float(u[q * 4 + 3]));
        return;
    }
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        pk[i] = zero ? 0u : pack_bf16(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1]));
    __nv_bfloat16* const dst[4] = {drow[0] ? drow[0] + col0 : nullptr, drow[1] ? drow[1] + col0 : nullptr,
                                   drow[2] ? drow[2] + col0 : nullptr, drow[3] ? drow[3] + col0 : nullptr};
    warp_store_chunk_pre(stage, pk, dst, ncols, lane);
}

__device__ __forceinline__ void epilogue_dw(const Params& p, const Tile& x, uint32_t tacc, int row, int half,
                                            uint32_t stage, int lane) {
    const int m = x.m0 + row;
    const bool live = m < p.dw_M;
    const int Mh = p.dw_M / 2;
    __nv_bfloat16* orow = nullptr;
    float* frow = nullptr;
    if (live) {
        if (p.dw_kind == 0) orow = p.dw_out0 + ((size_t)x.g * p.dw_M + m) * p.dw_N;
        else if (p.dw_kind == 1) orow = m < Mh ? p.dw_out0 + ((size_t)x.g * Mh + m) * p.dw_N
                                               : p.dw_out1 + ((size_t)x.g * Mh + m - Mh) * p.dw_N;
        else frow = p.dw_out_f32 + ((size_t)x.g * p.dw_M + m) * p.dw_N;
    }
    // destinations of the transposed stores: rows sg * 8 + lane / 4 of this warp's 32 rows
    __nv_bfloat16* drow[4];
#pragma unroll
    for (int sg = 0; sg < 4; ++sg)
        drow[sg] = reinterpret_cast<__nv_bfloat16*>(
            __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(orow), sg * 8 + (lane >> 2)));
    uint32_t ua[32], ub[32];
    const int c0 = half * 4;
    tmem_ld32(tacc + c0 * 32, ua);
    tmem_wait_ld();
    tmem_ld32(tacc + (c0 + 1) * 32, ub);
    dw_chunk(p, x, ua, c0, m, live, Mh, orow, frow, drow, stage, lane);
    tmem_wait_ld();
    tmem_ld32(tacc + (c0 + 2) * 32, ua);
    dw_chunk(p, x, ub, c0 + 1, m, live, Mh, orow, frow, drow, stage, lane);
    tmem_wait_ld();
    tmem_ld32(tacc + (c0 + 3) * 32, ub);
    dw_chunk(p, x, ua, c0 + 2, m, live, Mh, orow, frow, drow, stage, lane);
    tmem_wait_ld();
    dw_chunk(p, x, ub, c0 + 3, m, live, Mh, orow, frow, drow, stage, lane);
}

// DW, a tile of a group without rows (dw_zero): the producer thread writes its gradient block
// as zeros with TMA stores from the zeroed shared-memory block (32 rows per store), and the bias
// gradient rows of the tile that holds the bias column with bulk copies; M, M/2 and N are
// multiples of 32 rows / 64 columns, so no store crosses from one output matrix into the next.
__device__ __forceinline__ void dw_zero_tile(const Params& p, const Tile& x, uint32_t zbuf) {
    const int Mh = p.dw_M / 2;
    const bool bias_tile = p.dw_bias_col >= 0 && x.n0 <= p.dw_N && p.dw_N < x.n0 + 256;
    for (int rb = 0; rb < 4; ++rb) {
        const int m = x.m0 + 32 * rb;
        if (m >= p.dw_M) break;
        const bool hi = p.dw_kind == 1 && m >= Mh;
        const CUtensorMap* map = &p.tmZ[hi ? 1 : 0];
        const int y = p.dw_kind == 1 ? x.g * Mh + (hi ? m - Mh : m) : x.g * p.dw_M + m;
        for (int c = x.n0; c < x.n0 + 256 && c < p.dw_N; c += p.dw_zbw) tma_store_2d(map, zbuf, c, y);
        if (bias_tile) {
            __nv_bfloat16* b = p.dw_kind == 1 ? (hi ? p.dw_bias1 : p.dw_bias0) + (size_t)x.g * Mh + (hi ? m - Mh : m)
                                              : p.dw_bias0 + (size_t)x.g * p.dw_M + m;
            bulk_store(b, zbuf, 32 * 2);
        }
    }
    bulk_commit();
}

// ------------------------------------------------------------------------------ the kernel
// Pair protocol (expert GEMMs): both CTAs of a cluster pair run the same roles.  Each CTA's
// producer waits on its own "empty" barriers and loads its halves of A and B into its own
// ring, completing on the leader's "full" barrier; only the leader expects the pair's bytes,
// issues the MMAs (reading both CTAs' rings) and commits stages and accumulators to the
// barriers of both CTAs.  Each CTA's epilogue reads its own TMEM rows and arrives on the
// leader's "accumulator empty" barrier.  A cluster barrier after set-up makes the leader's
// barriers valid before any peer copy lands, and one before teardown keeps every shared
// memory and TMEM range alive until the leader's last MMA has finished.
//
// Q8 (GEMM1 / GEMM2R, single CTAs or pairs): routed tiles read e4m3 operands, K blocks of 128
// (the same 128-byte swizzle rows as 64 bf16), and run kind::f8f6f4 MMAs; shared-expert tiles
// of the same launch stay bf16.
template <int MODE, int KMAX, bool PAIR_, bool Q8 = false>
__global__ void __launch_bounds__(THREADS, 1) moe_tc_kernel(const __grid_constant__ Params p) {
    static_assert(!Q8 || MODE == GEMM1 || MODE == GEMM2R, "e4m3 tiles: routed expert GEMMs only");
    using C = Cfg<MODE, PAIR_>;
    constexpr bool PAIR = C::PAIR;
    constexpr int STAGES = C::STAGES;
    constexpr int B_BYTES = C::B_BYTES;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = base + STAGES * A_BYTES;
    const uint32_t bar0 = base + RING_BYTES;
    // barrier addresses (8 bytes each)
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
    auto ovl_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 5 + a); };   // mxw: shared columns drained
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + RING_BYTES + 8 * (2 * STAGES + 7));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    static_assert(8 * (2 * STAGES + 7) + 8 <= 256, "barrier area");
    static_assert(!Q8 || PAIR || STAGES <= 4, "scale-byte ring sized for 4 stages");
    // mxw: the stages' B and A scale bytes, after the epilogue buffers
    const uint32_t sf_base = bar0 + 256 + EPI_WARPS * STAGE_OUT_BYTES;
    auto sfb_stage = [&](int s) { return sf_base + (uint32_t)(s * SF_STAGE_BYTES); };
    auto sfa_stage = [&](int s) { return sf_base + (uint32_t)(4 * SF_STAGE_BYTES + s * SFA_BYTES); };
    const bool mxw = Q8 && !PAIR && p.mxw;
    const uint32_t acc_cols = mxw ? (uint32_t)(ACC_COLS - MX_OVL) : (uint32_t)ACC_COLS;   // second accumulator's start

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = PAIR ? cluster_rank() : 0u;        // 0 = leader of the pair
    const bool leader = rank == 0;
    const int cta_slot = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;   // pair index
    const int cta_slots = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), PAIR ? 2 * EPI_WARPS : EPI_WARPS);
            mbar_init(ovl_bar(a), EPI_WARPS / 2);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    const uint32_t zbuf = bar0 + 256 + EPI_WARPS * STAGE_OUT_BYTES;   // DW: ZERO_BYTES of zeros
    if (MODE == DW && p.dw_zero) {
        for (int i = threadIdx.x; i < ZERO_BYTES / 16; i += THREADS)
            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(zbuf + 16u * i), "r"(0u) : "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the TMA stores
    }
    if (warp == 1) {
        if (PAIR) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                         "r"(TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                         "r"(TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int ntiles = total_tiles<MODE, PAIR>(p);

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            if (MODE != GEMM1 || p.g_begin < p.E) prefetch_map(&p.tmA[0]);
            prefetch_map(&p.tmB[0]);
            int stage = 0;
            uint32_t phase = 0;
            int last_parity[STAGES];
#pragma unroll
            for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
            bool ok = true;
            const int arow = (int)rank * BM;                 // this CTA's rows inside a pair tile
            for (int t = cta_slot; ok && t < ntiles; t += cta_slots) {
                const Tile x = decode<MODE, PAIR>(p, t);
                if (MODE == DW && p.dw_zero && x.num_kb == 0) {
                    dw_zero_tile(p, x, zbuf);
                    continue;
                }
                // DW: a tile holding only the bias column loads one 64-column box of B (N = 64 MMAs)
                const int nbox = (MODE == DW && x.n0 >= p.dw_N) ? 1 : 4;
                for (int kk_ = 0; kk_ < x.num_kb; ++kk_) {
                    const int kb = x.kb0 + kk_;
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.err)) { ok = false; break; }
                    const uint32_t fb = full_bar(stage);
                    const uint32_t a_dst = sA + stage * A_BYTES, b_dst = sB + stage * B_BYTES;
                    if (MODE == ROUTER || MODE == ROUTERP) {
                        mbar_expect_tx(fb, A_BYTES + p.n_mma * BK * 2);
                        tma_load_2d(a_dst, &p.tmA[0], fb, kb * BK, x.m0);
                        tma_load_2d(b_dst, &p.tmB[0], fb, kb * BK, 0);
                    } else if (PAIR) {
                        if (leader) mbar_expect_tx(fb, 2 * (A_BYTES + B_BYTES));
                        if (MODE == GEMM1) {
                            // leader: W1 rows n0..n0+127 (accumulator columns 0-127);
                            // follower: the same rows of W3 (columns 128-255)
                            const bool shared = x.g >= p.E;
                            const int e = shared ? x.g - p.E : x.g;
                            const int kc = kb * ((Q8 && !shared) ? 2 * BK : BK);   // K element offset
                            tma_load_2d_pair(a_dst, &p.tmA[shared ? 1 : 0], fb, kc, x.row0 + x.m0 + arow);
                            tma_load_3d_pair(b_dst, &p.tmB[(shared ? 2 : 0) + (int)rank], fb, kc, x.n0, e);
                        } else if (MODE == GEMM2R && x.g >= 0) {
                            const int kc = kb * (Q8 ? 2 * BK : BK);
                            tma_load_2d_pair(a_dst, &p.tmA[0], fb, kc, x.row0 + x.m0 + arow);
                            tma_load_3d_pair(b_dst, &p.tmB[0], fb, kc, x.n0 + arow, x.g);
                        } else if (MODE == GEMM2R) {
                            const int kbs = ceil_div(p.Is, BK);
                            const int s = kb / kbs, kk = kb % kbs;
                            tma_load_3d_pair(a_dst, &p.tmA[1], fb, kk * BK, x.m0 + arow, s);
                            tma_load_3d_pair(b_dst, &p.tmB[1], fb, kk * BK, x.n0 + arow, s);
                        } else {
                            const int kbs = ceil_div(p.Is, BK);
                            const int s = kb / kbs, kk = kb % kbs;
                            tma_load_3d_pair(a_dst, &p.tmA[0], fb, kk * BK, x.m0 + arow, s);
                            tma_load_3d_pair(b_dst, &p.tmB[0], fb, kk * BK, x.n0 + arow, s);
                        }
                    } else if (MODE == DH || MODE == DX || MODE == DXS || MODE == DW) {
                        // MN-major B: four 64-column boxes of BK rows, 8 KB apart; DW's A likewise (two)
                        mbar_expect_tx(fb, A_BYTES + ((MODE == DW && !p.mn_wide) ? nbox * 8192 : B_BYTES));
                        if (MODE == DH) {
                            const bool shared = x.g >= p.E;
                            const int e = shared ? x.g - p.E : x.g;
                            tma_load_2d(a_dst, &p.tmA[shared ? 1 : 0], fb, kb * BK, x.row0 + x.m0);
                            if (p.mn_wide) tma_load_4d(b_dst, &p.tmB[shared ? 1 : 0], fb, 0, kb * BK, x.n0 / 64, e);
                            else
#pragma unroll
                                for (int j = 0; j < 4; ++j)
                                    tma_load_3d(b_dst + j * 8192, &p.tmB[shared ? 1 : 0], fb, x.n0 + 64 * j, kb * BK, e);
                        } else if (MODE == DX) {
                            const int kbh = ceil_div(p.I, BK);
                            const int hb = kb >= kbh ? 1 : 0;                  // 0: da . W1, 1: dg . W3
                            tma_load_2d(a_dst, &p.tmA[0], fb, kb * BK, x.row0 + x.m0);
                            if (p.mn_wide) tma_load_4d(b_dst, &p.tmB[hb], fb, 0, (kb - hb * kbh) * BK, x.n0 / 64, x.g);
                            else
#pragma unroll
                                for (int j = 0; j < 4; ++j)
                                    tma_load_3d(b_dst + j * 8192, &p.tmB[hb], fb, x.n0 + 64 * j, (kb - hb * kbh) * BK,
                                                x.g);
                        } else if (MODE == DXS) {
                            const int kbs = 2 * ceil_div(p.Is, BK);
                            if (kb < p.Ks * kbs) {
                                const int sx = kb / kbs, kk = kb % kbs;
                                const int hb = kk >= kbs / 2 ? 1 : 0;
                                tma_load_3d(a_dst, &p.tmA[0], fb, kk * BK, x.m0, sx);
                                if (p.mn_wide)
                                    tma_load_4d(b_dst, &p.tmB[hb], fb, 0, (kk - hb * (kbs / 2)) * BK, x.n0 / 64, sx);
                                else
#pragma unroll
                                    for (int j = 0; j < 4; ++j)
                                        tma_load_3d(b_dst + j * 8192, &p.tmB[hb], fb, x.n0 + 64 * j,
                                                    (kk - hb * (kbs / 2)) * BK, sx);
                            } else {
                                const int kr = kb - p.Ks * kbs;            // router: dz . C
                                tma_load_2d(a_dst, &p.tmA[1], fb, kr * BK, x.m0);
                                if (p.mn_wide) tma_load_4d(b_dst, &p.tmB[2], fb, 0, kr * BK, x.n0 / 64, 0);
                                else
#pragma unroll
                                    for (int j = 0; j < 4; ++j)
                                        tma_load_2d(b_dst + j * 8192, &p.tmB[2], fb, x.n0 + 64 * j, kr * BK);
                            }
                        } else if (p.mn_wide) {
                            // the 2 (A) and 4 (B) 64-column blocks of the stage in one request each,
                            // block j landing 8 KB after block j - 1 as with separate boxes
                            const int kr = x.row0 + kb * BK;
                            tma_load_4d(a_dst, &p.tmA[1], fb, 0, p.dw_a3d ? kb * BK : kr, x.m0 / 64, p.dw_a3d ? x.g : 0);
                            tma_load_4d(b_dst, &p.tmB[1], fb, 0, p.dw_b3d ? kb * BK : kr, x.n0 / 64, p.dw_b3d ? x.g : 0);
                        } else {
                            const int kr = x.row0 + kb * BK;
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                if (p.dw_a3d) tma_load_3d(a_dst + j * 8192, &p.tmA[0], fb, x.m0 + 64 * j, kb * BK, x.g);
                                else tma_load_2d(a_dst + j * 8192, &p.tmA[0], fb, x.m0 + 64 * j, kr);
                            }
                            for (int j = 0; j < nbox; ++j) {
                                if (p.dw_b3d) tma_load_3d(b_dst + j * 8192, &p.tmB[0], fb, x.n0 + 64 * j, kb * BK, x.g);
                                else tma_load_2d(b_dst + j * 8192, &p.tmB[0], fb, x.n0 + 64 * j, kr);
                            }
                        }
                    } else {
                        // block-scaled e4m3 tile: the stage's B (1 KB) and A (512 B) scale bytes come along
                        const bool sf_tile = mxw && (MODE == GEMM1 ? x.g < p.E : (MODE == GEMM2R && x.g >= 0));
                        mbar_expect_tx(fb, A_BYTES + B_BYTES + (sf_tile ? SF_STAGE_BYTES + SFA_BYTES : 0));
                        if (sf_tile) {
                            const uint8_t* src =
                                MODE == GEMM1
                                    ? p.sf13 + (((size_t)x.g * ceil_div(p.I, 128) + x.n0 / 128) * ceil_div(p.d, 128) + kb) *
                                                   SF_STAGE_BYTES
                                    : p.sf2 + (((size_t)x.g * ceil_div(p.d, 256) + x.n0 / 256) * ceil_div(p.I, 128) + kb) *
                                                  SF_STAGE_BYTES;
                            bulk_load(sfb_stage(stage), src, SF_STAGE_BYTES, fb);
                            bulk_load(sfa_stage(stage), p.sfa + ((size_t)mx_mtile<MODE>(p, x) * x.num_kb + kb) * SFA_BYTES,
                                      SFA_BYTES, fb);
                        }
                        if (MODE == GEMM1) {
                            const bool shared = x.g >= p.E;
                            const int e = shared ? x.g - p.E : x.g;
                            const int kc = kb * ((Q8 && !shared) ? 2 * BK : BK);   // K element offset
                            tma_load_2d(a_dst, &p.tmA[shared ? 1 : 0], fb, kc, x.row0 + x.m0);
                            if (p.w13_one & (shared ? 2 : 1)) {         // W3's block lands B_BYTES / 2 after W1's
                                tma_load_4d(b_dst, &p.tmB[shared ? 2 : 0], fb, kc, x.n0, 0, e);
                            } else {
                                tma_load_3d(b_dst, &p.tmB[shared ? 2 : 0], fb, kc, x.n0, e);
                                tma_load_3d(b_dst + B_BYTES / 2, &p.tmB[shared ? 3 : 1], fb, kc, x.n0, e);
                            }
                        } else if (MODE == GEMM2R && x.g >= 0) {
                            const int kc = kb * (Q8 ? 2 * BK : BK);
                            tma_load_2d(a_dst, &p.tmA[0], fb, kc, x.row0 + x.m0);
                            tma_load_3d(b_dst, &p.tmB[0], fb, kc, x.n0, x.g);
                        } else if (MODE == GEMM2R) {
                            const int kbs = ceil_div(p.Is, BK);
                            const int s = kb / kbs, kk = kb % kbs;
                            tma_load_3d(a_dst, &p.tmA[1], fb, kk * BK, x.m0, s);
                            tma_load_3d(b_dst, &p.tmB[1], fb, kk * BK, x.n0, s);
                        } else {
                            const int kbs = ceil_div(p.Is, BK);
                            const int s = kb / kbs, kk = kb % kbs;
                            tma_load_3d(a_dst, &p.tmA[0], fb, kk * BK, x.m0, s);
                            tma_load_3d(b_dst, &p.tmB[0], fb, kk * BK, x.n0, s);
                        }
                    }
                    last_parity[stage] = (int)phase;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // drain: every copy this thread issued has landed before the CTA may exit.  The
            // leader sees the pair's bytes on its own full barriers; a follower knows its copies
            // landed once the leader's MMA has released the stage they filled.
#pragma unroll
            for (int s = 0; s < STAGES; ++s) {
                if (last_parity[s] < 0) continue;
                if (leader) mbar_wait(full_bar(s), (uint32_t)last_parity[s], abort_flag, p.err, false);
                else mbar_wait(empty_bar(s), (uint32_t)last_parity[s], abort_flag, p.err, false);
            }
            if (MODE == DW && p.dw_zero) bulk_wait_all();   // zero stores done before the block is freed
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0 && leader) {
            const uint32_t idesc = PAIR ? idesc_bf16_pair(p.n_mma) : idesc_bf16(p.n_mma);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = cta_slot; ok && t < ntiles; t += cta_slots) {
                const Tile x = decode<MODE, PAIR>(p, t);
                if (MODE == DW && p.dw_zero && x.num_kb == 0) continue;      // written by the producer
                const bool q8tile = Q8 && (MODE == GEMM1 ? x.g < p.E : x.g >= 0);
                constexpr bool B_MN = MODE == DH || MODE == DX || MODE == DXS || MODE == DW;
                constexpr bool A_MN = MODE == DW;
                const bool narrow = MODE == DW && x.n0 >= p.dw_N;             // bias column only
                const uint32_t idesc_t = q8tile ? (PAIR ? idesc_e4m3_pair(p.n_mma) : idesc_e4m3(p.n_mma))
                                       : narrow ? idesc_bf16(64) | IDESC_B_MN | IDESC_A_MN
                                                : idesc | (B_MN ? IDESC_B_MN : 0u) | (A_MN ? IDESC_A_MN : 0u);
                if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.err)) break;
                // mxw: the previous tile (other accumulator) has drained the columns both share
                if (mxw && !mbar_wait(ovl_bar(acc ^ 1), acc ? acc_phase : acc_phase ^ 1u, abort_flag, p.err)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * acc_cols;
                const bool sf_tile = mxw && q8tile;
                for (int kb = 0; kb < x.num_kb; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag, p.err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = sA + stage * A_BYTES, b_addr = sB + stage * B_BYTES;
                    if (sf_tile) {
                        // this stage's scales: A rows -> columns SFA_COL..+3; B rows 0-127 -> SFB_COL..+3,
                        // rows 128-255 -> SFB_COL + 4..+7
                        tmem_cp_sf(tmem_base + SFA_COL, sf_desc(sfa_stage(stage)));
                        tmem_cp_sf(tmem_base + SFB_COL, sf_desc(sfb_stage(stage)));
                        tmem_cp_sf(tmem_base + SFB_COL + 4, sf_desc(sfb_stage(stage) + 512));
                    }
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        const uint64_t ad = A_MN ? mn_sw128_desc(a_addr + k * 2048) : sw128_desc(a_addr + k * 32);
                        const uint64_t bd = B_MN ? mn_sw128_desc(b_addr + k * 2048) : sw128_desc(b_addr + k * 32);
                        const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
                        if (sf_tile)   // run k of the stage's four runs of 32: scale byte k
                            mma_mx(d_tmem, ad, bd, idesc_mx(p.n_mma, k), tmem_base + SFA_COL + ((uint32_t)k << 30),
                                   tmem_base + SFB_COL + ((uint32_t)k << 30), accum);
                        else if (PAIR && q8tile) mma_e4m3_pair(d_tmem, ad, bd, idesc_t, accum);
                        else if (PAIR) mma_bf16_pair(d_tmem, ad, bd, idesc_t, accum);
                        else if (q8tile) mma_e4m3(d_tmem, ad, bd, idesc_t, accum);
                        else mma_bf16(d_tmem, ad, bd, idesc_t, accum);
                    }
                    if (PAIR) mma_commit_pair_both(empty_bar(stage));
                    else mma_commit(empty_bar(stage));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                if (PAIR) mma_commit_pair_both(tfull_bar(acc));
                else mma_commit(tfull_bar(acc));
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            // drain: all MMAs issued by this thread have completed before TMEM is freed
            if (PAIR) mma_commit_pair_local(drain_bar);
            else mma_commit(drain_bar);
            mbar_wait(drain_bar, 0, abort_flag, p.err, false);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ epilogue
        const int quad = warp & 3;                  // TMEM lanes 32*quad .. 32*quad+31
        const uint32_t stage_out = bar0 + 256 + (warp - 2) * STAGE_OUT_BYTES;   // this warp's transpose buffer
        const int half = (warp - 2) / 4;            // which half of the columns (0 or 1)
        const int row = (int)rank * BM + quad * 32 + lane;   // row inside the (pair) tile
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = cta_slot; t < ntiles; t += cta_slots) {
            const Tile x = decode<MODE, PAIR>(p, t);
            if (MODE == DW && p.dw_zero && x.num_kb == 0) continue;          // written by the producer
            if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag, p.err)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)acc * acc_cols;
            // mxw: accumulator 0 shares its last chunk (half 1's), accumulator 1 its first (half 0's)
            const bool ovl_owner = mxw && half == (acc == 0 ? 1 : 0);
            const uint32_t ovl = ovl_owner ? ovl_bar(acc) : 0u;
            const bool ovl_last = ovl_owner && acc == 0;
            if (MODE == ROUTER) {
                if (half == 0) epilogue_router<KMAX>(p, x, tacc, row);
            } else if (MODE == ROUTERP) {
                epilogue_router_partial(p, x, tacc, row, half);
            } else if (MODE == GEMM1) {
                epilogue_gemm1<Q8>(p, x, tacc, row, half, stage_out, lane, ovl, ovl_last);
            } else if (MODE == GEMM2R) {
                if (x.g >= 0) epilogue_gemm2r<Q8>(p, x, tacc, row, half, stage_out, lane, ovl, ovl_last);
                else epilogue_gemm2s(p, x, tacc, row, half, ovl, lane, ovl_last);
            } else if (MODE == DH) {
                epilogue_dh(p, x, tacc, row, half, stage_out, lane);
            } else if (MODE == DX) {
                epilogue_dx(p, x, tacc, row, half, stage_out, lane);
            } else if (MODE == DW) {
                epilogue_dw(p, x, tacc, row, half, stage_out, lane);
            } else {
                epilogue_gemm2s(p, x, tacc, row, half);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR) mbar_arrive_rank0(tempty_bar(acc));
                else mbar_arrive(tempty_bar(acc));
            }
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        if (PAIR)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                         : "memory");
    }
}

// Self-test of the bounded wait (the path a pipeline takes when a barrier is never completed):
// one warp allocates tensor memory as the pipeline does, thread 0 initialises an mbarrier that
// nothing arrives at and waits on it through mbar_wait_limit; the wait can only end by giving up
// (error bit 2).  Then the warp frees the tensor memory and the kernel returns; out (if given):
// out[0] = 1 if the wait gave up (0 if it somehow completed), out[1] = the ns it waited.
__global__ void __launch_bounds__(32, 1) wait_selftest_kernel(unsigned long long limit_ns, uint32_t* err,
                                                              unsigned long long* out) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tmem_holder;
    __shared__ int abort_flag;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_holder)),
                 "r"(32)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
    __syncwarp();
    tc_fence_after();
    if (threadIdx.x == 0) {
        const unsigned long long t0 = globaltimer();
        const bool done = mbar_wait_limit(b, 0, &abort_flag, err, true, limit_ns);
        if (out) {
            out[0] = done ? 0ull : 1ull;
            out[1] = globaltimer() - t0;
        }
    }
    tc_fence_before();
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_holder), "r"(32) : "memory");
}

// ------------------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
    }
    return fn;
}

// bf16 tensor [outer][mid][inner] (mid = 1 for 2-D) with a box of box_inner x box_mid (x 1)
bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t mid, uint64_t outer, uint32_t box_inner,
              uint32_t box_mid, bool three_d) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {inner, mid, outer};
    cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
    cuuint32_t box[3] = {box_inner, box_mid, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, three_d ? 3 : 2, const_cast<void*>(ptr), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// bf16 matrix [outer][rows][ld] read MN-major: the 4-D view {64 columns, rows, ld / 64 column
// blocks, outer} (strides ld * 2, 128, rows * ld * 2 bytes) with a box of 64 x box_rows x nblk x 1,
// so that one request brings nblk consecutive 64-column blocks, each a 128B-swizzled
// [box_rows][64] block, 8 KB apart in shared memory.  ld must be a multiple of 64.
bool make_map_mn(CUtensorMap* m, const void* ptr, uint64_t ld, uint64_t rows, uint64_t outer, uint32_t box_rows,
                 uint32_t nblk) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || ld % 64) return false;
    cuuint64_t dims[4] = {64, rows, ld / 64, outer};
    cuuint64_t strides[3] = {ld * 2, 128, rows * ld * 2};
    cuuint32_t box[4] = {64, box_rows, nblk, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// W1 and W3 stacks [E][I][d] (esz-byte elements) at a fixed positive distance, e.g. the two
// halves of one [2][E][I][d] buffer: the 4-D view {d, I, 2, E} whose third coordinate selects W1
// or W3, with a box of box_k x 128 rows x 2, brings a tile's 128 rows of both in one request (W3's
// rows 128 * box_k * esz bytes after W1's, as two separate boxes would land).  False when the
// distance does not fit the view (the caller then loads the two blocks separately).
bool make_map_w13(CUtensorMap* m, const void* w1, const void* w3, uint64_t d, uint64_t I, uint64_t E, uint32_t box_k,
                  bool u8) {
    EncodeTiledFn fn = encode_fn();
    const long long gap = (long long)((const char*)w3 - (const char*)w1);
    if (!fn || gap <= 0 || gap % 16 || gap >= (1ll << 40)) return false;
    const uint64_t esz = u8 ? 1 : 2;
    cuuint64_t dims[4] = {d, I, 2, E};
    cuuint64_t strides[3] = {d * esz, (cuuint64_t)gap, I * d * esz};
    cuuint32_t box[4] = {box_k, 128, 2, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(w1),
                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// bf16 matrix [rows][inner] as the target of TMA stores: box box_inner x box_rows, no swizzle
bool make_store_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_inner,
                    uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// e4m3 (byte) tensor [outer][mid][inner] with a box of box_inner x box_mid (x 1); inner must
// be a multiple of 16 (16-byte strides)
bool make_map_u8(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t mid, uint64_t outer, uint32_t box_inner,
                 uint32_t box_mid, bool three_d) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || inner % 16) return false;
    cuuint64_t dims[3] = {inner, mid, outer};
    cuuint64_t strides[2] = {inner, inner * mid};
    cuuint32_t box[3] = {box_inner, box_mid, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, three_d ? 3 : 2, const_cast<void*>(ptr), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Launches MODE.  Pair modes run as clusters of 2 CTAs; `tiles` bounds the useful CTAs (pairs
// for pair modes), and the grid never exceeds what can be resident at once (persistent loop).
template <int MODE, int KMAX, bool PAIR = false, bool Q8 = false>
cudaError_t launch(const Params& p, int tiles, cudaStream_t stream) {
    auto kern = moe_tc_kernel<MODE, KMAX, PAIR, Q8>;
    constexpr int smem = MODE == DW ? SMEM_BYTES_DW : (Q8 && !PAIR) ? SMEM_BYTES_Q8 : SMEM_BYTES;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    if (Cfg<MODE, PAIR>::PAIR) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        static int max_pairs = 0;
        if (!max_pairs) {
            cfg.gridDim = dim3(2 * (num_sms() / 2));
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = num_sms() / 2;
            max_pairs = n;
        }
        const int pairs = tiles < max_pairs ? (tiles > 0 ? tiles : 1) : max_pairs;
        cfg.gridDim = dim3(2 * pairs);
    } else {
        const int grid = tiles < num_sms() ? (tiles > 0 ? tiles : 1) : num_sms();
        cfg.gridDim = dim3(grid);
    }
    e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

Params base_params(const Dims& D, uint32_t* err) {
    Params p;
    memset(&p, 0, sizeof(p));
    p.T = D.T; p.d = D.d; p.E = D.E; p.I = D.I; p.Is = D.Ks > 0 ? D.Is : 8; p.k = D.k; p.Ks = D.Ks;
    p.S = D.slots();
    p.n_mma = 256;
    p.group_m = MOE_GROUP_M;
    p.err = err;
    return p;
}

}  // namespace tc

cudaError_t launch_wait_selftest(unsigned long long limit_ns, uint32_t* err, unsigned long long* out,
                                 cudaStream_t stream) {
    tc::wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, err, out);
    return cudaGetLastError();
}

int num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

// Whether the expert GEMMs run on CTA pairs.  Measured on one B200 with both variants
// interleaved, single CTAs are faster or equal for every layer shape here: bf16 prefill 14.3 vs
// 15.0 ms per layer, decode 3.9 vs 5.8 ms, mid 0.73 vs 0.77 ms; e4m3 routed experts, prefill
// 10.2 vs 10.3 ms (GEMM1 5.07 vs 5.15 ms, clock-normalised), although a pair reads 8 KB of
// operands per SM for each 256 x 256 x 32 e4m3 step where a single CTA reads 12 KB per
// 128 x 256 x 32.  Pairs (bf16 and e4m3 tiles, both parity-tested) stay available through a
// build with MOE_PAIR_POLICY=1.
bool gemm_pairs(const Dims& D) {
    (void)D;
#if defined(MOE_PAIR_POLICY) && MOE_PAIR_POLICY > 0
    return !D.mx;                          // block-scaled tiles run on single CTAs only
#else
    return false;
#endif
}
namespace tc {
bool pairs_for(const Dims& D) { return gemm_pairs(D); }
}

bool tc_router_supported(const Dims& D) { return D.bf16 && D.E % 16 == 0 && D.E >= 16 && D.E <= 256; }

int router_splits(const Dims& D) {
    if (!tc_router_supported(D) || D.T == 0) return 1;
    const int mt = ceil_div(D.T, tc::BM);
    const int kbt = ceil_div(D.d, tc::BK);
    if (mt > 32 || kbt < 16) return 1;
    constexpr int kCtas = 148;                       // fixed so the workspace size never depends on the GPU
    const int want = ceil_div(kCtas, mt);
    const int per = ceil_div(kbt, want < kbt ? want : kbt);
    return ceil_div(kbt, per < 4 ? 4 : per);
}

cudaError_t launch_tc_router(const Dims& D, const void* x, const void* centroids, const float* bias, int32_t* idx,
                             float* gate, float* partial, uint32_t* err, cudaStream_t stream) {
    using namespace tc;
    if (D.T == 0) return cudaSuccess;
    Params p = base_params(D, err);
    p.n_mma = D.E;
    p.idx_out = idx;
    p.gate_out = gate;
    p.router_bias = bias;
    p.gate_mode = D.gate_mode;
    if (!make_map(&p.tmA[0], x, D.d, D.T, 1, BK, BM, false)) return cudaErrorInvalidValue;
    if (!make_map(&p.tmB[0], centroids, D.d, D.E, 1, BK, D.E, false)) return cudaErrorInvalidValue;
    const int mt = ceil_div(D.T, BM);
    const int nsplit = router_splits(D);
    if (nsplit > 1 && partial) {
        const int kbt = ceil_div(D.d, BK);
        p.kb_per_split = ceil_div(kbt, nsplit);
        p.partial = partial;
        const int tiles = mt * ceil_div(kbt, p.kb_per_split);
        cudaError_t e = launch<ROUTERP, 8>(p, tiles, stream);
        if (e != cudaSuccess) return e;
        return launch_router_finish(D, partial, ceil_div(kbt, p.kb_per_split), bias, idx, gate, stream);
    }
    return D.k <= 8 ? launch<ROUTER, 8>(p, mt, stream) : launch<ROUTER, 32>(p, mt, stream);
}

cudaError_t launch_tc_gemm1(const Dims& D, const void* x, const void* x_perm, const int32_t* offsets,
                            const int32_t* tile_start1, const FfnWeights& R, const FfnWeights& Sh, void* h_r, void* h_s,
                            int g_begin, int g_end, uint32_t* err, cudaStream_t stream, const SavedAG* save) {
    using namespace tc;
    if (D.T == 0 || g_end <= g_begin) return cudaSuccess;
    Params p = base_params(D, err);
    if (save) {
        p.a_out = (__nv_bfloat16*)save->a; p.g_out = (__nv_bfloat16*)save->g;
        p.as_out = (__nv_bfloat16*)save->as; p.gs_out = (__nv_bfloat16*)save->gs;
    }
    p.tile_start = tile_start1;
    p.offsets = offsets;
    p.g_begin = g_begin;
    p.g_end = g_end;
    p.b1 = (const __nv_bfloat16*)R.b1; p.b3 = (const __nv_bfloat16*)R.b3;
    p.sb1 = (const __nv_bfloat16*)Sh.b1; p.sb3 = (const __nv_bfloat16*)Sh.b3;
    p.h_r = (__nv_bfloat16*)h_r; p.h_s = (__nv_bfloat16*)h_s;
    bool ok = true;
    if (g_begin < D.E) {
        ok &= make_map(&p.tmA[0], x_perm, D.d, (uint64_t)D.slots(), 1, BK, BM, false);
        ok &= make_map(&p.tmB[0], R.w1, D.d, D.I, D.E, BK, 128, true);
        ok &= make_map(&p.tmB[1], R.w3, D.d, D.I, D.E, BK, 128, true);
    }
    if (g_end > D.E) {
        ok &= make_map(&p.tmA[1], x, D.d, D.T, 1, BK, BM, false);
        ok &= make_map(&p.tmB[2], Sh.w1, D.d, D.Is, D.Ks, BK, 128, true);
        ok &= make_map(&p.tmB[3], Sh.w3, D.d, D.Is, D.Ks, BK, 128, true);
    }
    if (!ok) return cudaErrorInvalidValue;
    if (!tc::pairs_for(D)) {                   // one request for both weight blocks where the layout allows
        CUtensorMap w;
        if (g_begin < D.E && make_map_w13(&w, R.w1, R.w3, D.d, D.I, D.E, BK, false)) { p.tmB[0] = w; p.w13_one |= 1; }
        if (g_end > D.E && make_map_w13(&w, Sh.w1, Sh.w3, D.d, D.Is, D.Ks, BK, false)) { p.tmB[2] = w; p.w13_one |= 2; }
    }
    // tile count lives on the device
    return tc::pairs_for(D) ? launch<GEMM1, 8, true>(p, num_sms(), stream) : launch<GEMM1, 8, false>(p, num_sms(), stream);
}

cudaError_t launch_tc_gemm2_routed(const Dims& D, const int32_t* offsets, const int32_t* tile_start2,
                                   const float* sorted_gate, const FfnWeights& R, const void* h_r, void* y_sorted,
                                   const FfnWeights* Sh, const void* h_s, float* sout, uint32_t* err,
                                   cudaStream_t stream) {
    using namespace tc;
    if (D.T == 0) return cudaSuccess;
    Params p = base_params(D, err);
    p.tile_start = tile_start2;
    p.offsets = offsets;
    p.sorted_gate = sorted_gate;
    p.b2 = (const __nv_bfloat16*)R.b2;
    p.y = (__nv_bfloat16*)y_sorted;
    const bool pairs = tc::pairs_for(D);
    bool ok = make_map(&p.tmA[0], h_r, D.I, (uint64_t)D.slots(), 1, BK, BM, false);
    ok &= make_map(&p.tmB[0], R.w2, D.I, D.d, D.E, BK, pairs ? 128 : 256, true);
    if (Sh && D.Ks > 0 && sout) {
        p.fold_shared = 1;
        p.sb2 = (const __nv_bfloat16*)Sh->b2;
        p.sout = sout;
        ok &= make_map(&p.tmA[1], h_s, D.Is, D.T, D.Ks, BK, BM, true);
        ok &= make_map(&p.tmB[1], Sh->w2, D.Is, D.d, D.Ks, BK, pairs ? 128 : 256, true);
    }
    if (!ok) return cudaErrorInvalidValue;
    return pairs ? launch<GEMM2R, 8, true>(p, num_sms(), stream)
                 : launch<GEMM2R, 8, false>(p, num_sms(), stream);
}

cudaError_t launch_tc_gemm2_shared(const Dims& D, const FfnWeights& Sh, const void* h_s, float* sout, uint32_t* err,
                                   cudaStream_t stream) {
    using namespace tc;
    if (D.T == 0 || D.Ks == 0) return cudaSuccess;
    Params p = base_params(D, err);
    p.sb2 = (const __nv_bfloat16*)Sh.b2;
    p.sout = sout;
    bool ok = make_map(&p.tmA[0], h_s, D.Is, D.T, D.Ks, BK, BM, true);
    ok &= make_map(&p.tmB[0], Sh.w2, D.Is, D.d, D.Ks, BK, tc::pairs_for(D) ? 128 : 256, true);
    if (!ok) return cudaErrorInvalidValue;
    const int n = ceil_div(D.d, 256);
    return tc::pairs_for(D) ? launch<GEMM2S, 8, true>(p, ceil_div(D.T, 256) * n, stream)
                         : launch<GEMM2S, 8, false>(p, ceil_div(D.T, 128) * n, stream);
}

// e4m3 routed experts: GEMM1 over x8_perm (e4m3 rows, one scale per row in xs) and the e4m3
// W1 / W3 codes with their channel scales; shared groups [E, g_end) stay bf16 on x.
cudaError_t launch_tc_gemm1_q8(const Dims& D, const void* x, const void* x8_perm, const float* xs,
                               const int32_t* offsets, const int32_t* tile_start1, const FfnWeights& R,
                               const FfnWeights& Sh, void* h_r, void* h_s, int g_end, uint32_t* err,
                               cudaStream_t stream, const MxAct* mx) {
    using namespace tc;
    if (D.T == 0) return cudaSuccess;
    if (D.mx ? (!R.sf13 || !mx || !mx->sfa || !mx->h8 || !mx->sfh) : (!R.s1 || !R.s3 || !xs))
        return cudaErrorInvalidValue;
    Params p = base_params(D, err);
    p.q8 = 1;
    p.a_scale = xs;
    p.ws1 = R.s1; p.ws3 = R.s3;
    p.mxw = D.mx ? 1 : 0;
    p.sf13 = R.sf13;
    if (D.mx) { p.sfa = mx->sfa; p.h8_out = mx->h8; p.sfh_out = mx->sfh; }
    const bool pairs = tc::pairs_for(D);                   // never for block scales (gemm_pairs)
    p.tile_start = tile_start1;
    p.offsets = offsets;
    p.g_begin = 0;
    p.g_end = g_end;
    p.b1 = (const __nv_bfloat16*)R.b1; p.b3 = (const __nv_bfloat16*)R.b3;
    p.sb1 = (const __nv_bfloat16*)Sh.b1; p.sb3 = (const __nv_bfloat16*)Sh.b3;
    p.h_r = (__nv_bfloat16*)h_r; p.h_s = (__nv_bfloat16*)h_s;
    bool ok = make_map_u8(&p.tmA[0], x8_perm, D.d, (uint64_t)D.slots(), 1, 2 * BK, BM, false);
    ok &= make_map_u8(&p.tmB[0], R.w1, D.d, D.I, D.E, 2 * BK, 128, true);
    ok &= make_map_u8(&p.tmB[1], R.w3, D.d, D.I, D.E, 2 * BK, 128, true);
    if (g_end > D.E) {
        ok &= make_map(&p.tmA[1], x, D.d, D.T, 1, BK, BM, false);
        ok &= make_map(&p.tmB[2], Sh.w1, D.d, D.Is, D.Ks, BK, 128, true);
        ok &= make_map(&p.tmB[3], Sh.w3, D.d, D.Is, D.Ks, BK, 128, true);
    }
    if (!ok) return cudaErrorInvalidValue;
    if (!pairs) {
        CUtensorMap w;
        if (make_map_w13(&w, R.w1, R.w3, D.d, D.I, D.E, 2 * BK, true)) { p.tmB[0] = w; p.w13_one |= 1; }
        if (g_end > D.E && make_map_w13(&w, Sh.w1, Sh.w3, D.d, D.Is, D.Ks, BK, false)) { p.tmB[2] = w; p.w13_one |= 2; }
    }
    return pairs ? launch<GEMM1, 8, true, true>(p, num_sms(), stream)
                 : launch<GEMM1, 8, false, true>(p, num_sms(), stream);
}

// e4m3 routed GEMM2 over h8 (e4m3 rows, scale per row in hs) and the e4m3 W2 codes; with Sh the
// shared experts' bf16 GEMM2 tiles follow in the same launch (-> sout), as in the bf16 path.
cudaError_t launch_tc_gemm2_routed_q8(const Dims& D, const int32_t* offsets, const int32_t* tile_start2,
                                      const float* sorted_gate, const FfnWeights& R, const void* h8,
                                      const float* hs, void* y_sorted, const FfnWeights* Sh, const void* h_s,
                                      float* sout, uint32_t* err, cudaStream_t stream, const MxAct* mx) {
    using namespace tc;
    if (D.T == 0) return cudaSuccess;
    if (D.mx ? (!R.sf2 || !mx || !mx->sfa) : (!R.s2 || !hs)) return cudaErrorInvalidValue;
    Params p = base_params(D, err);
    p.q8 = 1;
    p.a_scale = hs;
    p.ws2 = R.s2;
    p.mxw = D.mx ? 1 : 0;
    p.sf2 = R.sf2;
    if (D.mx) p.sfa = mx->sfa;
    p.tile_start = tile_start2;
    p.offsets = offsets;
    p.sorted_gate = sorted_gate;
    p.b2 = (const __nv_bfloat16*)R.b2;
    p.y = (__nv_bfloat16*)y_sorted;
    const bool pairs = tc::pairs_for(D);                   // never for block scales (gemm_pairs)
    bool ok = make_map_u8(&p.tmA[0], h8, D.I, (uint64_t)D.slots(), 1, 2 * BK, BM, false);
    ok &= make_map_u8(&p.tmB[0], R.w2, D.I, D.d, D.E, 2 * BK, pairs ? 128 : 256, true);
    if (Sh && D.Ks > 0 && sout) {
        p.fold_shared = 1;
        p.sb2 = (const __nv_bfloat16*)Sh->b2;
        p.sout = sout;
        ok &= make_map(&p.tmA[1], h_s, D.Is, D.T, D.Ks, BK, BM, true);
        ok &= make_map(&p.tmB[1], Sh->w2, D.Is, D.d, D.Ks, BK, pairs ? 128 : 256, true);
    }
    if (!ok) return cudaErrorInvalidValue;
    return pairs ? launch<GEMM2R, 8, true, true>(p, num_sms(), stream)
                 : launch<GEMM2R, 8, false, true>(p, num_sms(), stream);
}

// ------------------------------------------------------------------------------ backward
// fp32 router logits z = x . C^T [T][N_m] (the split-K router's partial-logit mode with one split)
cudaError_t launch_router_logits(const Dims& D, const void* x, const void* centroids, float* z, uint32_t* err,
                                 cudaStream_t stream) {
    using namespace tc;
    if (D.T == 0) return cudaSuccess;
    if (!tc_router_supported(D)) return cudaErrorInvalidValue;
    Params p = base_params(D, err);
    p.n_mma = D.E;
    p.partial = z;
    p.kb_per_split = ceil_div(D.d, BK);
    if (!make_map(&p.tmA[0], x, D.d, D.T, 1, BK, BM, false)) return cudaErrorInvalidValue;
    if (!make_map(&p.tmB[0], centroids, D.d, D.E, 1, BK, D.E, false)) return cudaErrorInvalidValue;
    return launch<ROUTERP, 8>(p, ceil_div(D.T, BM), stream);
}

cudaError_t launch_tc_dh(const Dims& D, const BwdBufs& B, const FfnWeights& R, const FfnWeights& Sh, const void* dout,
                         uint32_t* err, cudaStream_t stream) {
    using namespace tc;
    if (D.T == 0) return cudaSuccess;
    Params p = base_params(D, err);
    p.tile_start = B.ts_dh;
    p.offsets = B.offsets;
    p.offs_pad = B.offs_pad;
    p.sorted_gate = B.sorted_gate;
    p.a_sv = (const __nv_bfloat16*)B.a_sv; p.g_sv = (const __nv_bfloat16*)B.g_sv;
    p.as_sv = (const __nv_bfloat16*)B.as_sv; p.gs_sv = (const __nv_bfloat16*)B.gs_sv;
    p.dag = (__nv_bfloat16*)B.dag; p.hg = (__nv_bfloat16*)B.hg;
    p.dag_s = (__nv_bfloat16*)B.dag_s; p.hg_s = (__nv_bfloat16*)B.hg_s;
    p.dgate_part = B.dgate_part;
    p.n_parts = 2 * ceil_div(D.I, 256);
    bool ok = make_map(&p.tmA[0], B.dout_pad, D.d, (uint64_t)B.S_pad, 1, BK, BM, false);
    ok &= make_map(&p.tmB[0], R.w2, D.I, D.d, D.E, 64, BK, true);
    if (D.Ks > 0) {
        ok &= make_map(&p.tmA[1], dout, D.d, D.T, 1, BK, BM, false);
        ok &= make_map(&p.tmB[1], Sh.w2, D.Is, D.d, D.Ks, 64, BK, true);
    }
    if (!ok) return cudaErrorInvalidValue;
    CUtensorMap w[2];
    if (make_map_mn(&w[0], R.w2, D.I, D.d, D.E, BK, 4) && (D.Ks == 0 || make_map_mn(&w[1], Sh.w2, D.Is, D.d, D.Ks, BK, 4))) {
        p.tmB[0] = w[0];
        if (D.Ks > 0) p.tmB[1] = w[1];
        p.mn_wide = 1;
    }
    return launch<DH, 8>(p, num_sms(), stream);
}

cudaError_t launch_tc_dx(const Dims& D, const BwdBufs& B, const FfnWeights& R, uint32_t* err, cudaStream_t stream) {
    using namespace tc;
    if (D.T == 0) return cudaSuccess;
    Params p = base_params(D, err);
    p.tile_start = B.ts_dx;
    p.offsets = B.offsets;
    p.offs_pad = B.offs_pad;
    p.dx_slot = (__nv_bfloat16*)B.dx_slot;
    bool ok = make_map(&p.tmA[0], B.dag, 2 * (uint64_t)D.I, (uint64_t)B.S_pad, 1, BK, BM, false);
    ok &= make_map(&p.tmB[0], R.w1, D.d, D.I, D.E, 64, BK, true);
    ok &= make_map(&p.tmB[1], R.w3, D.d, D.I, D.E, 64, BK, true);
    if (!ok) return cudaErrorInvalidValue;
    CUtensorMap w[2];
    if (make_map_mn(&w[0], R.w1, D.d, D.I, D.E, BK, 4) && make_map_mn(&w[1], R.w3, D.d, D.I, D.E, BK, 4)) {
        p.tmB[0] = w[0];
        p.tmB[1] = w[1];
        p.mn_wide = 1;
    }
    return launch<DX, 8>(p, num_sms(), stream);
}

cudaError_t launch_tc_dxs(const Dims& D, const BwdBufs& B, const FfnWeights& Sh, const void* centroids, uint32_t* err,
                          cudaStream_t stream) {
    using namespace tc;
    if (D.T == 0) return cudaSuccess;
    Params p = base_params(D, err);
    p.sout = B.base;
    p.sb2 = nullptr;
    bool ok = make_map(&p.tmA[1], B.dz_bf16, D.E, D.T, 1, BK, BM, false);
    ok &= make_map(&p.tmB[2], centroids, D.d, D.E, 1, 64, BK, false);
    if (D.Ks > 0) {
        ok &= make_map(&p.tmA[0], B.dag_s, 2 * (uint64_t)D.Is, D.T, D.Ks, BK, BM, true);
        ok &= make_map(&p.tmB[0], Sh.w1, D.d, D.Is, D.Ks, 64, BK, true);
        ok &= make_map(&p.tmB[1], Sh.w3, D.d, D.Is, D.Ks, 64, BK, true);
    } else {                                   // keep every map the kernel prefetches valid
        ok &= make_map(&p.tmA[0], B.dz_bf16, D.E, D.T, 1, BK, BM, false);
        ok &= make_map(&p.tmB[0], centroids, D.d, D.E, 1, 64, BK, false);
    }
    if (!ok) return cudaErrorInvalidValue;
    CUtensorMap w[3];
    if (make_map_mn(&w[2], centroids, D.d, D.E, 1, BK, 4) &&
        (D.Ks > 0 ? make_map_mn(&w[0], Sh.w1, D.d, D.Is, D.Ks, BK, 4) && make_map_mn(&w[1], Sh.w3, D.d, D.Is, D.Ks, BK, 4)
                  : make_map_mn(&w[0], centroids, D.d, D.E, 1, BK, 4))) {
        p.tmB[0] = w[0];
        if (D.Ks > 0) p.tmB[1] = w[1];
        p.tmB[2] = w[2];
        p.mn_wide = 1;
    }
    return launch<DXS, 8>(p, ceil_div(D.T, BM) * ceil_div(D.d, 256), stream);
}

cudaError_t launch_tc_dw(const Dims& D, const DwSpec& w, uint32_t* err, cudaStream_t stream) {
    using namespace tc;
    if (w.groups <= 0 || w.M <= 0 || w.N <= 0) return cudaSuccess;
    Params p = base_params(D, err);
    p.dw_kind = w.kind;
    p.dw_groups = w.groups; p.dw_M = w.M; p.dw_N = w.N;
    p.dw_a3d = w.a3d; p.dw_b3d = w.b3d;
    p.dw_rows = w.rows;
    p.dw_K = w.K;
    p.dw_out0 = (__nv_bfloat16*)w.out0; p.dw_out1 = (__nv_bfloat16*)w.out1;
    p.dw_out_f32 = w.out_f32;
    // Raster: the smaller operand of a group stays in L2 while the larger streams once.  kind 0
    // (A = dout rows, d wide; B = gate * h, I wide): all N tiles of an M tile in a row; kinds 1, 2
    // (A = da | dg or dz, narrower than B = x): all M tiles of an N tile in a row.
    p.group_m = w.kind == 0 ? 1 : ceil_div(w.M, BM);
    p.dw_bias_col = w.bias0 ? w.N : -1;
    p.dw_Nt = w.bias0 ? w.N + 1 : w.N;
    p.dw_bias0 = (__nv_bfloat16*)w.bias0; p.dw_bias1 = (__nv_bfloat16*)w.bias1;
    const int b_ld = w.b_ld > 0 ? w.b_ld : w.N;
    if (w.bias0 && b_ld < w.N + 1) return cudaErrorInvalidValue;
    bool ok = make_map(&p.tmA[0], w.a, (uint64_t)w.M, (uint64_t)w.a_rows, w.a3d ? w.groups : 1, 64, BK, w.a3d);
    ok &= make_map(&p.tmB[0], w.b, (uint64_t)b_ld, (uint64_t)w.b_rows, w.b3d ? w.groups : 1, 64, BK, w.b3d);
    // one request per operand and stage where both widths are whole 64-column blocks (the view
    // must not reach past a row's end), else one request per 64-column block
    if (w.M % 64 == 0 && b_ld % 64 == 0)
        p.mn_wide = make_map_mn(&p.tmA[1], w.a, (uint64_t)w.M, (uint64_t)w.a_rows, w.a3d ? w.groups : 1, BK, 2) &&
                    make_map_mn(&p.tmB[1], w.b, (uint64_t)b_ld, (uint64_t)w.b_rows, w.b3d ? w.groups : 1, BK, 4);
    if (w.rows && w.kind != 2) {
        // groups may be empty: their bf16 gradients (and bias gradients) are zero-filled by the
        // producer's TMA stores, 32 rows x up to 256 columns each
        const int Mo = w.kind == 1 ? w.M / 2 : w.M;
        auto a16 = [](const void* q) { return ((uintptr_t)q & 15u) == 0; };
        if (w.N % 64 || Mo % 32 || !a16(w.out0) || (w.kind == 1 && !a16(w.out1)) || (w.bias0 && !a16(w.bias0)) ||
            (w.bias1 && !a16(w.bias1)))
            return cudaErrorInvalidValue;
        p.dw_zero = 1;
        p.dw_zbw = w.N < 256 ? w.N : 256;
        ok &= make_store_map(&p.tmZ[0], w.out0, (uint64_t)w.N, (uint64_t)w.groups * Mo, p.dw_zbw, 32);
        if (w.kind == 1) ok &= make_store_map(&p.tmZ[1], w.out1, (uint64_t)w.N, (uint64_t)w.groups * Mo, p.dw_zbw, 32);
    }
    if (!ok) return cudaErrorInvalidValue;
    const long long tiles = (long long)w.groups * ceil_div(w.M, BM) * ceil_div(p.dw_Nt, 256);
    return launch<DW, 8>(p, (int)(tiles < num_sms() ? tiles : num_sms()), stream);
}

}  // namespace moe
