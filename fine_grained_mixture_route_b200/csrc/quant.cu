// Per-row e4m3 quantisation of bf16 rows: the activation side of the FP8 routed experts.
//
// For every output row p (source row r = row_of[p], or p): scale[p] = max_j |src[r, j]| / 448
// (1 for an all-zero row) and dst[p, j] = e4m3(src[r, j] / scale[p]), where the division is
// IEEE fp32 and e4m3() rounds to the nearest e4m3 value, ties to even, saturating at +-448.
// 448 is the largest finite e4m3 value, so the row maximum lands on it.  The same steps on the
// same fp32 values give the same codes on any IEEE machine, which makes the quantised rows
// reproducible bit for bit.
#include <cuda_fp8.h>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float chunk_amax(const uint4& v, float m) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
    return m;
}

// 8 bf16 -> 8 e4m3 codes (element j in byte j)
__device__ __forceinline__ uint2 chunk_quant(const uint4& v, float sc) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = make_float2(__fdiv_rn(bf16_lo(w[i]), sc), __fdiv_rn(bf16_hi(w[i]), sc));
        pk[i] = (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
    }
    return make_uint2(pk[0] | (pk[1] << 16), pk[2] | (pk[3] << 16));
}

// One warp per row, the whole row in registers (CPL 16-byte chunks per lane): loads of a row
// are all issued before the reduction, and no block barrier sits between rows.
template <int CPL>
__global__ void __launch_bounds__(256) quant_rows_warp_kernel(const uint4* __restrict__ src,
                                                              const int32_t* __restrict__ row_of, long long n_rows,
                                                              int src_rows, int nv, uint2* __restrict__ dst,
                                                              float* __restrict__ scale, uint32_t* err) {
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long p = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < n_rows; p += warps) {
        int r = row_of ? row_of[p] : (int)p;
        const bool ok = r >= 0 && r < src_rows;
        if (!ok) {
            if (lane == 0) flag_error(err, ERR_INDEX_RANGE);
            r = 0;
        }
        const uint4* s = src + (size_t)r * nv;
        uint4 keep[CPL];
        float m = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int i = lane + c * 32;
            keep[c] = (ok && i < nv) ? __ldg(s + i) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int c = 0; c < CPL; ++c) m = chunk_amax(keep[c], m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float sc = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
        if (lane == 0) scale[p] = sc;
        uint2* d = dst + (size_t)p * nv;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int i = lane + c * 32;
            if (i < nv) d[i] = chunk_quant(keep[c], sc);
        }
    }
}

// One warp per row for rows wider than the register-resident kernels take: the row is read
// twice, in batches of 8 chunks per lane (the second pass finds it in L1 / L2).
__global__ void __launch_bounds__(256) quant_rows_warp2_kernel(const uint4* __restrict__ src,
                                                               const int32_t* __restrict__ row_of, long long n_rows,
                                                               int src_rows, int nv, uint2* __restrict__ dst,
                                                               float* __restrict__ scale, uint32_t* err) {
    constexpr int B = 8;
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long p = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < n_rows; p += warps) {
        int r = row_of ? row_of[p] : (int)p;
        const bool ok = r >= 0 && r < src_rows;
        if (!ok) {
            if (lane == 0) flag_error(err, ERR_INDEX_RANGE);
            r = 0;
        }
        const uint4* s = src + (size_t)r * nv;
        float m = 0.f;
        for (int base = 0; ok && base < nv; base += 32 * B) {
            uint4 v[B];
#pragma unroll
            for (int c = 0; c < B; ++c) {
                const int i = base + lane + c * 32;
                v[c] = i < nv ? __ldg(s + i) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int c = 0; c < B; ++c) m = chunk_amax(v[c], m);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float sc = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
        if (lane == 0) scale[p] = sc;
        uint2* d = dst + (size_t)p * nv;
        for (int base = 0; base < nv; base += 32 * B) {
            uint4 v[B];
#pragma unroll
            for (int c = 0; c < B; ++c) {
                const int i = base + lane + c * 32;
                v[c] = (ok && i < nv) ? __ldg(s + i) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int c = 0; c < B; ++c) {
                const int i = base + lane + c * 32;
                if (i < nv) d[i] = chunk_quant(v[c], sc);
            }
        }
    }
}

template <int CPL>
cudaError_t launch_warp(const void* src, const int32_t* row_of, long long n_rows, int src_rows, int nv, uint8_t* dst,
                        float* scale, uint32_t* err, cudaStream_t stream) {
    const long long cap = (long long)num_sms() * 8;                 // 8 blocks of 8 warps per SM at most
    const long long need = (n_rows + 7) / 8;
    quant_rows_warp_kernel<CPL><<<(int)(need < cap ? need : cap), 256, 0, stream>>>(
        (const uint4*)src, row_of, n_rows, src_rows, nv, (uint2*)dst, scale, err);
    return cudaGetLastError();
}

// dst[p] = src[row_of[p]] for rows of `row_bytes` bytes (a multiple of 16), and, when given,
// dscale[p] = sscale[row_of[p]]; one block per row per grid-stride step.
__global__ void gather_code_rows_kernel(const uint4* __restrict__ src, const float* __restrict__ sscale,
                                        const int32_t* __restrict__ row_of, long long n_rows, int src_rows, int nv,
                                        uint4* __restrict__ dst, float* __restrict__ dscale, uint32_t* err) {
    for (long long p = blockIdx.x; p < n_rows; p += gridDim.x) {
        const int r = row_of[p];
        const bool ok = r >= 0 && r < src_rows;
        if (!ok && threadIdx.x == 0) flag_error(err, ERR_INDEX_RANGE);
        const uint4* s = src + (size_t)(ok ? r : 0) * nv;
        uint4* d = dst + (size_t)p * nv;
        for (int i = threadIdx.x; i < nv; i += blockDim.x) d[i] = ok ? __ldg(s + i) : make_uint4(0, 0, 0, 0);
        if (dscale && threadIdx.x == 0) dscale[p] = ok ? sscale[r] : 1.f;
    }
}

// Token-order form of the same move: dst[slot_of[t*k + j]] = src[t] (and its scale) for every
// pick j of row t, so each source row is read once and stored k times.  A position outside
// [0, S) sets bit 4 and is skipped; a dropped slot (-1) is skipped.
__global__ void scatter_code_rows_kernel(const uint4* __restrict__ src, const float* __restrict__ sscale,
                                         const int32_t* __restrict__ slot_of, int T, int k, long long S, int nv,
                                         uint4* __restrict__ dst, float* __restrict__ dscale, uint32_t* err) {
    __shared__ int pos[32];
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();
        if ((int)threadIdx.x < k) {
            int q = slot_of[(size_t)t * k + threadIdx.x];
            if (q >= S) { flag_error(err, ERR_INDEX_RANGE); q = -1; }
            pos[threadIdx.x] = q;
            if (q >= 0 && dscale) dscale[q] = sscale[t];
        }
        __syncthreads();
        const uint4* s = src + (size_t)t * nv;
        for (int i = threadIdx.x; i < nv; i += blockDim.x) {
            const uint4 v = __ldg(s + i);
            for (int j = 0; j < k; ++j)
                if (pos[j] >= 0) dst[(size_t)pos[j] * nv + i] = v;
        }
    }
}

// dst[p] = src[row_of[p]] for rows of nw 4-byte words (16-byte vectors when nw % 4 == 0); an
// index outside [0, src_rows) sets bit 4 and gives a zero row.
template <bool V16>
__global__ void gather_rows_generic_kernel(const uint32_t* __restrict__ src, const int32_t* __restrict__ row_of,
                                           long long n_rows, long long src_rows, int nw, uint32_t* __restrict__ dst,
                                           uint32_t* err) {
    const int nv = V16 ? nw / 4 : nw;
    for (long long p = blockIdx.x; p < n_rows; p += gridDim.x) {
        const long long r = row_of[p];
        const bool ok = r >= 0 && r < src_rows;
        if (!ok && threadIdx.x == 0) flag_error(err, ERR_INDEX_RANGE);
        if (V16) {
            const uint4* s = reinterpret_cast<const uint4*>(src) + (size_t)(ok ? r : 0) * nv;
            uint4* d = reinterpret_cast<uint4*>(dst) + (size_t)p * nv;
            for (int i = threadIdx.x; i < nv; i += blockDim.x) d[i] = ok ? __ldg(s + i) : make_uint4(0, 0, 0, 0);
        } else {
            const uint32_t* s = src + (size_t)(ok ? r : 0) * nv;
            uint32_t* d = dst + (size_t)p * nv;
            for (int i = threadIdx.x; i < nv; i += blockDim.x) d[i] = ok ? __ldg(s + i) : 0u;
        }
    }
}

// ids[r] = q % modulo for the segment q that holds row r, the segments being consecutive runs
// of counts[q] rows.  Every block scans the (at most SEGMENT_MAX) counts into shared memory,
// then finds the segment of each of its rows by binary search over the segment starts.  A
// negative count is taken as 0 and a row past the last segment gets -1; both set bit 4.
constexpr int SEG_THREADS = 256;
__global__ void __launch_bounds__(SEG_THREADS) segment_ids_kernel(const int32_t* __restrict__ counts, int n_seg,
                                                                  int modulo, long long n_rows,
                                                                  int32_t* __restrict__ ids, uint32_t* err) {
    __shared__ long long start[SEGMENT_MAX + 1];
    __shared__ long long chunk[SEG_THREADS];
    const int per = (n_seg + SEG_THREADS - 1) / SEG_THREADS;
    const int b = threadIdx.x * per, e = min(n_seg, b + per);
    long long run = 0;
    for (int q = b; q < e; ++q) {
        const int c = counts[q];
        if (c < 0 && blockIdx.x == 0) flag_error(err, ERR_INDEX_RANGE);
        start[q] = run;                          // local start inside this thread's chunk
        run += c > 0 ? c : 0;
    }
    chunk[threadIdx.x] = run;
    __syncthreads();
    if (threadIdx.x == 0) {                      // exclusive scan of the 256 chunk sums
        long long acc = 0;
        for (int i = 0; i < SEG_THREADS; ++i) {
            const long long v = chunk[i];
            chunk[i] = acc;
            acc += v;
        }
        start[n_seg] = acc;
    }
    __syncthreads();
    for (int q = b; q < e; ++q) start[q] += chunk[threadIdx.x];
    __syncthreads();
    const long long total = start[n_seg];
    for (long long r = (long long)blockIdx.x * SEG_THREADS + threadIdx.x; r < n_rows;
         r += (long long)gridDim.x * SEG_THREADS) {
        if (r >= total) {
            ids[r] = -1;
            flag_error(err, ERR_INDEX_RANGE);
            continue;
        }
        int lo = 0, hi = n_seg;                  // largest q with start[q] <= r: start[lo] <= r < start[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (start[mid] <= r) lo = mid;
            else hi = mid;
        }
        ids[r] = lo % modulo;
    }
}

}  // namespace

cudaError_t launch_gather_rows_generic(const void* src, const int32_t* row_of, long long n_rows, long long src_rows,
                                       int row_bytes, void* dst, uint32_t* err, cudaStream_t stream) {
    if (n_rows <= 0) return cudaSuccess;
    if (row_bytes <= 0 || row_bytes % 4) return cudaErrorInvalidValue;
    const int nw = row_bytes / 4;
    const bool v16 = nw % 4 == 0 && ((uintptr_t)src & 15u) == 0 && ((uintptr_t)dst & 15u) == 0;
    const int threads = nw >= 512 ? 128 : 32;
    const long long cap = (long long)num_sms() * 16;
    const int blocks = (int)(n_rows < cap ? n_rows : cap);
    if (v16)
        gather_rows_generic_kernel<true><<<blocks, threads, 0, stream>>>((const uint32_t*)src, row_of, n_rows, src_rows,
                                                                         nw, (uint32_t*)dst, err);
    else
        gather_rows_generic_kernel<false><<<blocks, threads, 0, stream>>>((const uint32_t*)src, row_of, n_rows,
                                                                          src_rows, nw, (uint32_t*)dst, err);
    return cudaGetLastError();
}

namespace {

// ---- block-scaled e4m3 weights (MOE_FMT_MXFP8) ---------------------------------------
// Each weight row (one output channel, K inputs) is cut into runs of 32 consecutive inputs; a
// run's scale is 2^e with e the smallest integer such that max|run| <= 448 * 2^e (no element
// saturates), 0 for an all-zero run, within [-127, 127]; the codes are e4m3(v * 2^-e), the
// product exact (a power of two), rounded to nearest even.  The scale is stored as the byte
// e + 127, in the tiled order the GEMMs' pipeline stages load (see mx_scale_offset).

// 8 bf16 times a power of two -> 8 e4m3 codes (element j in byte j)
__device__ __forceinline__ uint2 chunk_quant_mul(const uint4& v, float mul) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = make_float2(bf16_lo(w[i]) * mul, bf16_hi(w[i]) * mul);
        pk[i] = (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
    }
    return make_uint2(pk[0] | (pk[1] << 16), pk[2] | (pk[3] << 16));
}

// Byte offset of the scale of run j of row r of expert e in the tiled layout: rows in groups of
// P (128 for W1 / W3, 256 for W2), runs in chunks of 4 (one pipeline stage of 128 inputs); the
// 1 KB block of (e, group, chunk) holds two 512-byte halves (W1 / W3: half = which matrix;
// W2: half = (r / 128) % 2), and in a half row r's byte for run j sits at
// (r % 32) * 16 + ((r / 32) % 4) * 4 + j % 4.
__device__ __forceinline__ size_t mx_scale_offset(int e, int r, int j, int ngrp, int nch, int P, int which) {
    const size_t blk = ((size_t)e * ngrp + r / P) * nch + j / 4;
    const int half = P == 128 ? which : (r / 128) & 1;
    return blk * 1024 + half * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (j & 3);
}

// One warp per row; lane i of a pass holds 16-byte chunk i (8 elements), so lanes 4q..4q+3 hold
// run q of the pass and two shuffles give its maximum.  P > 0: weight scales in the tiled order;
// P == 0: activation rows, row q's scale of run j at sf[q * ceil(K / 32) + j].
__global__ void __launch_bounds__(256) quant_weights_mx_kernel(const uint4* __restrict__ src, int E, int rows, int K,
                                                               int P, int which, uint2* __restrict__ codes,
                                                               uint8_t* __restrict__ sf) {
    const int lane = threadIdx.x & 31;
    const int nv = K / 8;
    const int nch = (K + 127) / 128;
    const int nruns = (K + 31) / 32;
    const int ngrp = P > 0 ? (rows + P - 1) / P : 0;
    const long long n_rows = (long long)E * rows;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long q = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); q < n_rows; q += warps) {
        const int e = (int)(q / rows), r = (int)(q % rows);
        const uint4* s = src + (size_t)q * nv;
        uint2* dst = codes + (size_t)q * nv;
        for (int base = 0; base < nv; base += 32) {
            const int i = base + lane;
            const uint4 v = i < nv ? s[i] : make_uint4(0u, 0u, 0u, 0u);
            float m = chunk_amax(v, 0.f);
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            const int ex = mx_exponent(m);
            const float mul = __uint_as_float((uint32_t)(127 - ex) << 23);   // 2^-ex (ex <= 126 for finite runs)
            if (i < nv) dst[i] = chunk_quant_mul(v, mul);
            if ((lane & 3) == 0 && i < nv)
                sf[P > 0 ? mx_scale_offset(e, r, i >> 2, ngrp, nch, P, which) : (size_t)q * nruns + (i >> 2)] =
                    (uint8_t)(ex + 127);
        }
    }
}

// The A-side scales of the block-scaled GEMM1: grouped position p (token stok[p], in expert e's
// rows [offsets[e], offsets[e + 1])) is row r = (p - offsets[e]) % 128 of the expert's 128-row
// block m = (p - offsets[e]) / 128, whose global index is tile_start1[e] / n_tiles + m.  One warp
// per position finds e (binary search over the offsets, every lane on the same addresses), then
// lane l copies the token's scale bytes of runs 4c..4c+3 (127 past the row) for chunks
// c = l, l + 32, ... to the block's chunk c: [M-tile][chunk][512], row r at (r % 32) * 16 +
// (r / 32 % 4) * 4.
__global__ void __launch_bounds__(256) scatter_sf_tiled_kernel(
    const uint8_t* __restrict__ xsf, int nruns, const int32_t* __restrict__ stok, int T,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ tile_start1, int E, long long S, int n_tiles,
    int nch, uint8_t* __restrict__ sfa, uint32_t* err) {
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long p = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < S; p += warps) {
        const int t = stok[p];
        if (t < 0 || t >= T) {
            if (lane == 0) flag_error(err, ERR_INDEX_RANGE);
            continue;
        }
        int lo = 0, hi = E;                               // the last e with offsets[e] <= p
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (offsets[mid] <= p) lo = mid;
            else hi = mid - 1;
        }
        const int local = (int)(p - offsets[lo]);
        const size_t base = (size_t)(tile_start1[lo] / n_tiles + local / 128) * nch * 512 + (local & 31) * 16 +
                            ((local >> 5) & 3) * 4;
        const uint8_t* row = xsf + (size_t)t * nruns;
        for (int c = lane; c < nch; c += 32) {
            uint32_t w = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int run = 4 * c + q;
                w |= (uint32_t)(run < nruns ? row[run] : 127u) << (8 * q);
            }
            *reinterpret_cast<uint32_t*>(sfa + base + (size_t)c * 512) = w;
        }
    }
}

}  // namespace

size_t mx_act_scale_bytes(long long slots, int n_experts, int K) {
    return (size_t)((slots + 127) / 128 + n_experts) * ((K + 127) / 128) * 512;
}

cudaError_t launch_quant_rows_mx(const void* src, int rows, int K, uint8_t* codes, uint8_t* sf, cudaStream_t stream) {
    if (rows <= 0) return cudaSuccess;
    if (K % 8) return cudaErrorInvalidValue;
    const long long cap = 8LL * 8 * num_sms();
    const int blocks = (int)((rows + 7) / 8 < cap ? (rows + 7) / 8 : cap);
    quant_weights_mx_kernel<<<blocks, 256, 0, stream>>>((const uint4*)src, 1, rows, K, 0, 0, (uint2*)codes, sf);
    return cudaGetLastError();
}

cudaError_t launch_scatter_sf_tiled(const uint8_t* xsf, int T, int K, const int32_t* stok, const int32_t* offsets,
                                    const int32_t* tile_start1, int E, long long S, int I, uint8_t* sfa, uint32_t* err,
                                    cudaStream_t stream) {
    if (S <= 0) return cudaSuccess;
    const int nch = (K + 127) / 128;
    const long long cap = 8LL * 8 * num_sms();
    const int blocks = (int)((S + 7) / 8 < cap ? (S + 7) / 8 : cap);    // one warp per grouped position
    scatter_sf_tiled_kernel<<<blocks, 256, 0, stream>>>(xsf, (K + 31) / 32, stok, T, offsets, tile_start1, E, S,
                                                        (I + 127) / 128, nch, sfa, err);
    return cudaGetLastError();
}

size_t mx_scale_bytes(int kind, long long n_experts, int rows, int K) {
    const int P = kind == 0 ? 128 : 256;
    return (size_t)n_experts * ((rows + P - 1) / P) * ((K + 127) / 128) * 1024;
}

cudaError_t launch_quant_weights_mx(int kind, const void* w, int which, int n_experts, int rows, int K, uint8_t* codes,
                                    uint8_t* sf, cudaStream_t stream) {
    const long long n = (long long)n_experts * rows;
    if (n == 0) return cudaSuccess;
    const long long cap = 8LL * 8 * num_sms();
    const int blocks = (int)((n + 7) / 8 < cap ? (n + 7) / 8 : cap);
    quant_weights_mx_kernel<<<blocks, 256, 0, stream>>>((const uint4*)w, n_experts, rows, K, kind == 0 ? 128 : 256,
                                                        which, (uint2*)codes, sf);
    return cudaGetLastError();
}

cudaError_t launch_quant_rows(const void* src, const int32_t* row_of, long long n_rows, int src_rows, int width,
                              uint8_t* dst, float* scale, uint32_t* err, cudaStream_t stream) {
    if (n_rows <= 0) return cudaSuccess;
    if (width <= 0 || width % 8) return cudaErrorInvalidValue;
    const int nv = width / 8;
    if (nv <= 32) return launch_warp<1>(src, row_of, n_rows, src_rows, nv, dst, scale, err, stream);
    if (nv <= 64) return launch_warp<2>(src, row_of, n_rows, src_rows, nv, dst, scale, err, stream);
    if (nv <= 128) return launch_warp<4>(src, row_of, n_rows, src_rows, nv, dst, scale, err, stream);
    if (nv <= 256) return launch_warp<8>(src, row_of, n_rows, src_rows, nv, dst, scale, err, stream);
    const long long cap = (long long)num_sms() * 8;
    const long long need = (n_rows + 7) / 8;
    quant_rows_warp2_kernel<<<(int)(need < cap ? need : cap), 256, 0, stream>>>(
        (const uint4*)src, row_of, n_rows, src_rows, nv, (uint2*)dst, scale, err);
    return cudaGetLastError();
}

cudaError_t launch_gather_code_rows(const uint8_t* src, const float* sscale, const int32_t* row_of, long long n_rows,
                                    int src_rows, int row_bytes, uint8_t* dst, float* dscale, uint32_t* err,
                                    cudaStream_t stream) {
    if (n_rows <= 0) return cudaSuccess;
    if (row_bytes <= 0 || row_bytes % 16) return cudaErrorInvalidValue;
    const long long cap = (long long)num_sms() * 16;
    const int blocks = (int)(n_rows < cap ? n_rows : cap);
    gather_code_rows_kernel<<<blocks, 128, 0, stream>>>((const uint4*)src, sscale, row_of, n_rows, src_rows,
                                                        row_bytes / 16, (uint4*)dst, dscale, err);
    return cudaGetLastError();
}

cudaError_t launch_scatter_code_rows(const uint8_t* src, const float* sscale, const int32_t* slot_of, int T, int k,
                                     long long S, int row_bytes, uint8_t* dst, float* dscale, uint32_t* err,
                                     cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    if (row_bytes <= 0 || row_bytes % 16 || k > 32) return cudaErrorInvalidValue;
    const cudaError_t e = launch_scatter_rows_bulk(src, sscale, slot_of, T, k, S, (uint32_t)row_bytes, dst, dscale, err,
                                                   stream);
    if (e != cudaErrorNotSupported) return e;                  // else: the register copy below
    const int blocks = T < num_sms() * 16 ? T : num_sms() * 16;
    scatter_code_rows_kernel<<<blocks, 128, 0, stream>>>((const uint4*)src, sscale, slot_of, T, k, S, row_bytes / 16,
                                                         (uint4*)dst, dscale, err);
    return cudaGetLastError();
}

cudaError_t launch_segment_ids(const int32_t* counts, int n_seg, int modulo, long long n_rows, int32_t* ids,
                               uint32_t* err, cudaStream_t stream) {
    if (n_rows <= 0) return cudaSuccess;
    if (n_seg < 1 || n_seg > SEGMENT_MAX || modulo < 1) return cudaErrorInvalidValue;
    const long long need = (n_rows + SEG_THREADS - 1) / SEG_THREADS;
    const long long cap = (long long)num_sms() * 4;
    segment_ids_kernel<<<(int)(need < cap ? need : cap), SEG_THREADS, 0, stream>>>(counts, n_seg, modulo, n_rows, ids,
                                                                                  err);
    return cudaGetLastError();
}

}  // namespace moe
