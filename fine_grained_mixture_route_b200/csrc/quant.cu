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

constexpr int QT = 256;    // threads per row
constexpr int QREG = 4;    // 16-byte chunks per thread kept in registers between the passes

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

__global__ void __launch_bounds__(QT) quant_rows_kernel(const uint4* __restrict__ src,
                                                        const int32_t* __restrict__ row_of, long long n_rows,
                                                        int src_rows, int nv, uint2* __restrict__ dst,
                                                        float* __restrict__ scale, uint32_t* err) {
    __shared__ float red[QT / 32];
    const int tid = threadIdx.x;
    for (long long p = blockIdx.x; p < n_rows; p += gridDim.x) {
        int r = row_of ? row_of[p] : (int)p;
        const bool ok = r >= 0 && r < src_rows;
        if (!ok) {
            if (tid == 0) flag_error(err, ERR_INDEX_RANGE);
            r = 0;
        }
        const uint4* s = src + (size_t)r * nv;
        uint4 keep[QREG];
        float m = 0.f;
#pragma unroll
        for (int c = 0; c < QREG; ++c) {
            const int i = tid + c * QT;
            keep[c] = (ok && i < nv) ? __ldg(s + i) : make_uint4(0, 0, 0, 0);
            m = chunk_amax(keep[c], m);
        }
        for (int i = tid + QREG * QT; ok && i < nv; i += QT) m = chunk_amax(__ldg(s + i), m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        __syncthreads();                       // red[] of the previous row has been read
        if ((tid & 31) == 0) red[tid >> 5] = m;
        __syncthreads();
        float amax = red[0];
#pragma unroll
        for (int w = 1; w < QT / 32; ++w) amax = fmaxf(amax, red[w]);
        const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
        if (tid == 0) scale[p] = sc;
        uint2* d = dst + (size_t)p * nv;
#pragma unroll
        for (int c = 0; c < QREG; ++c) {
            const int i = tid + c * QT;
            if (i < nv) d[i] = chunk_quant(keep[c], sc);
        }
        for (int i = tid + QREG * QT; i < nv; i += QT) d[i] = ok ? chunk_quant(__ldg(s + i), sc) : make_uint2(0, 0);
    }
}

}  // namespace

cudaError_t launch_quant_rows(const void* src, const int32_t* row_of, long long n_rows, int src_rows, int width,
                              uint8_t* dst, float* scale, uint32_t* err, cudaStream_t stream) {
    if (n_rows <= 0) return cudaSuccess;
    if (width <= 0 || width % 8) return cudaErrorInvalidValue;
    const long long cap = (long long)num_sms() * 8;
    const int blocks = (int)(n_rows < cap ? n_rows : cap);
    quant_rows_kernel<<<blocks, QT, 0, stream>>>((const uint4*)src, row_of, n_rows, src_rows, width / 8,
                                                 (uint2*)dst, scale, err);
    return cudaGetLastError();
}

}  // namespace moe
