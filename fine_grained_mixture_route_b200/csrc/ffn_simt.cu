// CUDA-core grouped expert FFN for fp32 layers (the tiny fp32 configuration, where the
// 1e-4 tolerance rules out TF32 tensor cores).  Same math as the `Expert` module of
// "DeepSeek MoE模型优化与未来演进及字节超稀疏内存技术": h = silu(x w1^T + b1) * (x w3^T + b3),
// y = h w2^T + b2, with the routed outputs scaled by their gate and the shared experts and
// routed rows summed per token as in "《DeepSeekMoE》深度解读报告" §3.1.
//
// 64x64 output tiles, 16-deep K steps staged in shared memory, 4x4 outputs per thread.
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int FB_M = 64, FB_N = 64, FB_K = 16, FB_THREADS = 256;

template <typename T>
struct Ffn1Args {
    const T* x;
    const int32_t* offsets;
    const int32_t* sorted_token;
    const T *w1, *b1, *w3, *b3;       // routed stacks
    const T *sw1, *sb1, *sw3, *sb3;   // shared stacks
    T* h_r;
    T* h_s;
    int T_, d, E, I, Is, g_begin;
    long long S;
    uint32_t* err;
};

// GEMM1 + SwiGLU: grid (n-tiles of the hidden dim, m-tiles of T rows, groups)
template <typename T>
__global__ void __launch_bounds__(FB_THREADS) simt_gemm1_kernel(Ffn1Args<T> a) {
    __shared__ float As[FB_K][FB_M + 4];
    __shared__ float B1[FB_K][FB_N + 4];
    __shared__ float B3[FB_K][FB_N + 4];
    __shared__ int tok[FB_M];
    const int g = a.g_begin + blockIdx.z;
    const bool shared = g >= a.E;
    const int rows = shared ? a.T_ : a.offsets[g + 1] - a.offsets[g];
    const int row0 = shared ? 0 : a.offsets[g];
    const int I = shared ? a.Is : a.I;
    const int m0 = blockIdx.y * FB_M, n0 = blockIdx.x * FB_N;
    if (!shared && (row0 < 0 || rows < 0 || (long long)row0 + rows > a.S)) {   // offsets out of range
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) flag_error(a.err, ERR_INDEX_RANGE);
        return;
    }
    if (m0 >= rows || n0 >= I) return;
    const int e = shared ? g - a.E : g;
    const T* w1 = (shared ? a.sw1 : a.w1) + (size_t)e * I * a.d;
    const T* w3 = (shared ? a.sw3 : a.w3) + (size_t)e * I * a.d;
    const T* b1 = shared ? (a.sb1 ? a.sb1 + (size_t)e * I : nullptr) : (a.b1 ? a.b1 + (size_t)e * I : nullptr);
    const T* b3 = shared ? (a.sb3 ? a.sb3 + (size_t)e * I : nullptr) : (a.b3 ? a.b3 + (size_t)e * I : nullptr);
    const int tid = threadIdx.x;
    if (tid < FB_M) {
        int r = m0 + tid, t = -1;
        if (r < rows) {
            t = shared ? r : a.sorted_token[row0 + r];
            if (t < 0 || t >= a.T_) { flag_error(a.err, ERR_INDEX_RANGE); t = -1; }
        }
        tok[tid] = t;
    }
    __syncthreads();
    const int ty = tid / 16, tx = tid % 16;
    float acc1[4][4] = {}, acc3[4][4] = {};
    for (int k0 = 0; k0 < a.d; k0 += FB_K) {
        for (int i = tid; i < FB_M * FB_K; i += FB_THREADS) {
            int r = i / FB_K, c = i % FB_K, kk = k0 + c, t = tok[r];
            As[c][r] = (t >= 0 && kk < a.d) ? to_f32(a.x[(size_t)t * a.d + kk]) : 0.f;
            int n = n0 + r;
            bool okb = n < I && kk < a.d;
            B1[c][r] = okb ? to_f32(w1[(size_t)n * a.d + kk]) : 0.f;
            B3[c][r] = okb ? to_f32(w3[(size_t)n * a.d + kk]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < FB_K; ++c) {
            float av[4], bv1[4], bv3[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { av[i] = As[c][ty * 4 + i]; bv1[i] = B1[c][tx * 4 + i]; bv3[i] = B3[c][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc1[i][j] = fmaf(av[i], bv1[j], acc1[i][j]);
                    acc3[i][j] = fmaf(av[i], bv3[j], acc3[i][j]);
                }
        }
        __syncthreads();
    }
    T* h = shared ? a.h_s + (size_t)e * a.T_ * I : a.h_r + (size_t)row0 * I;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int r = m0 + ty * 4 + i;
        if (r >= rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int n = n0 + tx * 4 + j;
            if (n >= I) continue;
            float u = acc1[i][j] + (b1 ? to_f32(b1[n]) : 0.f);
            float v = acc3[i][j] + (b3 ? to_f32(b3[n]) : 0.f);
            h[(size_t)r * I + n] = from_f32<T>(silu_f32(u) * v);
        }
    }
}

template <typename T>
struct Ffn2Args {
    const int32_t* offsets;
    const float* sorted_gate;
    const T *w2, *b2;
    const T* h;
    T* y;
    // shared + combine
    const int32_t* slot_of;
    const T* y_sorted;
    T* out;
    int T_, d, E, I, k, Ks;
    long long S;
    uint32_t* err;
};

// MODE 0: routed GEMM2, y[p] = gate_p * (h[p] w2_e^T + b2_e); grid (n-tiles of d, m-tiles, E)
// MODE 1: shared GEMM2 accumulated over the K_s experts along K, plus the routed rows of each
//         token in ascending pick order; grid (n-tiles of d, m-tiles of T, 1)
template <typename T, int MODE>
__global__ void __launch_bounds__(FB_THREADS) simt_gemm2_kernel(Ffn2Args<T> a) {
    __shared__ float As[FB_K][FB_M + 4];
    __shared__ float Bs[FB_K][FB_N + 4];
    const int e = blockIdx.z;
    const int rows = MODE == 0 ? a.offsets[e + 1] - a.offsets[e] : a.T_;
    const int row0 = MODE == 0 ? a.offsets[e] : 0;
    const int m0 = blockIdx.y * FB_M, n0 = blockIdx.x * FB_N;
    if (MODE == 0 && (row0 < 0 || rows < 0 || (long long)row0 + rows > a.S)) {   // offsets out of range
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) flag_error(a.err, ERR_INDEX_RANGE);
        return;
    }
    if (m0 >= rows) return;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    float acc[4][4] = {};
    const int nexp = MODE == 0 ? 1 : a.Ks;
    for (int s = 0; s < nexp; ++s) {
        const int ex = MODE == 0 ? e : s;
        const T* w2 = a.w2 + (size_t)ex * a.d * a.I;
        const T* h = MODE == 0 ? a.h + (size_t)row0 * a.I : a.h + (size_t)s * a.T_ * a.I;
        for (int k0 = 0; k0 < a.I; k0 += FB_K) {
            for (int i = tid; i < FB_M * FB_K; i += FB_THREADS) {
                int r = i / FB_K, c = i % FB_K, kk = k0 + c;
                As[c][r] = (m0 + r < rows && kk < a.I) ? to_f32(h[(size_t)(m0 + r) * a.I + kk]) : 0.f;
                int n = n0 + r;
                Bs[c][r] = (n < a.d && kk < a.I) ? to_f32(w2[(size_t)n * a.I + kk]) : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int c = 0; c < FB_K; ++c) {
                float av[4], bv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) { av[i] = As[c][ty * 4 + i]; bv[i] = Bs[c][tx * 4 + i]; }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
            __syncthreads();
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = m0 + ty * 4 + i;
        if (r >= rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= a.d) continue;
            if (MODE == 0) {
                const int p = row0 + r;
                float v = acc[i][j] + (a.b2 ? to_f32(a.b2[(size_t)e * a.d + n]) : 0.f);
                const float g = a.sorted_gate ? a.sorted_gate[p] : 1.f;
                a.y[(size_t)p * a.d + n] = from_f32<T>(g * v);
            } else {
                float v = acc[i][j];
                if (a.b2)
                    for (int s = 0; s < a.Ks; ++s) v += to_f32(a.b2[(size_t)s * a.d + n]);
                for (int jj = 0; jj < a.k; ++jj) {
                    const int p = a.slot_of[(size_t)r * a.k + jj];
                    if (p < 0 || p >= a.S) { flag_error(a.err, ERR_INDEX_RANGE); continue; }
                    v += to_f32(a.y_sorted[(size_t)p * a.d + n]);
                }
                a.out[(size_t)r * a.d + n] = from_f32<T>(v);
            }
        }
    }
}

template <typename T>
cudaError_t gemm1_impl(const Dims& D, const void* x, const int32_t* offsets, const int32_t* sorted_token,
                       const FfnWeights& R, const FfnWeights& Sh, void* h_r, void* h_s, int g_begin, int g_end,
                       uint32_t* err, cudaStream_t stream) {
    Ffn1Args<T> a;
    a.x = (const T*)x; a.offsets = offsets; a.sorted_token = sorted_token;
    a.w1 = (const T*)R.w1; a.b1 = (const T*)R.b1; a.w3 = (const T*)R.w3; a.b3 = (const T*)R.b3;
    a.sw1 = (const T*)Sh.w1; a.sb1 = (const T*)Sh.b1; a.sw3 = (const T*)Sh.w3; a.sb3 = (const T*)Sh.b3;
    a.h_r = (T*)h_r; a.h_s = (T*)h_s;
    a.T_ = D.T; a.d = D.d; a.E = D.E; a.I = D.I; a.Is = D.Ks > 0 ? D.Is : 1; a.g_begin = g_begin; a.S = D.slots(); a.err = err;
    const int maxI = D.Ks > 0 && D.Is > D.I ? D.Is : D.I;
    dim3 grid(ceil_div(maxI, FB_N), ceil_div(D.T, FB_M), g_end - g_begin);
    if (grid.z == 0 || D.T == 0) return cudaSuccess;
    simt_gemm1_kernel<T><<<grid, FB_THREADS, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt_gemm1(const Dims& D, const void* x, const int32_t* offsets, const int32_t* sorted_token,
                              const FfnWeights& routed, const FfnWeights& shared, void* h_r, void* h_s, int g_begin,
                              int g_end, uint32_t* err, cudaStream_t stream) {
    if (D.bf16)
        return gemm1_impl<__nv_bfloat16>(D, x, offsets, sorted_token, routed, shared, h_r, h_s, g_begin, g_end, err,
                                         stream);
    return gemm1_impl<float>(D, x, offsets, sorted_token, routed, shared, h_r, h_s, g_begin, g_end, err, stream);
}

cudaError_t launch_simt_gemm2_routed(const Dims& D, const int32_t* offsets, const float* sorted_gate,
                                     const FfnWeights& routed, const void* h_r, void* y_sorted, uint32_t* err,
                                     cudaStream_t stream) {
    if (D.T == 0) return cudaSuccess;
    dim3 grid(ceil_div(D.d, FB_N), ceil_div(D.T, FB_M), D.E);
    if (D.bf16) {
        Ffn2Args<__nv_bfloat16> a = {};
        a.offsets = offsets; a.sorted_gate = sorted_gate;
        a.w2 = (const __nv_bfloat16*)routed.w2; a.b2 = (const __nv_bfloat16*)routed.b2;
        a.h = (const __nv_bfloat16*)h_r; a.y = (__nv_bfloat16*)y_sorted;
        a.T_ = D.T; a.d = D.d; a.E = D.E; a.I = D.I; a.k = D.k; a.S = D.slots(); a.err = err;
        simt_gemm2_kernel<__nv_bfloat16, 0><<<grid, FB_THREADS, 0, stream>>>(a);
    } else {
        Ffn2Args<float> a = {};
        a.offsets = offsets; a.sorted_gate = sorted_gate;
        a.w2 = (const float*)routed.w2; a.b2 = (const float*)routed.b2;
        a.h = (const float*)h_r; a.y = (float*)y_sorted;
        a.T_ = D.T; a.d = D.d; a.E = D.E; a.I = D.I; a.k = D.k; a.S = D.slots(); a.err = err;
        simt_gemm2_kernel<float, 0><<<grid, FB_THREADS, 0, stream>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_simt_gemm2_shared(const Dims& D, const FfnWeights& shared, const void* h_s, const void* y_sorted,
                                     const int32_t* slot_of, void* out, uint32_t* err, cudaStream_t stream) {
    if (D.T == 0) return cudaSuccess;
    dim3 grid(ceil_div(D.d, FB_N), ceil_div(D.T, FB_M), 1);
    if (D.bf16) {
        Ffn2Args<__nv_bfloat16> a = {};
        a.w2 = (const __nv_bfloat16*)shared.w2; a.b2 = (const __nv_bfloat16*)shared.b2;
        a.h = (const __nv_bfloat16*)h_s; a.slot_of = slot_of; a.y_sorted = (const __nv_bfloat16*)y_sorted;
        a.out = (__nv_bfloat16*)out;
        a.T_ = D.T; a.d = D.d; a.E = D.E; a.I = D.Is; a.k = D.k; a.Ks = D.Ks; a.S = D.slots(); a.err = err;
        simt_gemm2_kernel<__nv_bfloat16, 1><<<grid, FB_THREADS, 0, stream>>>(a);
    } else {
        Ffn2Args<float> a = {};
        a.w2 = (const float*)shared.w2; a.b2 = (const float*)shared.b2;
        a.h = (const float*)h_s; a.slot_of = slot_of; a.y_sorted = (const float*)y_sorted; a.out = (float*)out;
        a.T_ = D.T; a.d = D.d; a.E = D.E; a.I = D.Is; a.k = D.k; a.Ks = D.Ks; a.S = D.slots(); a.err = err;
        simt_gemm2_kernel<float, 1><<<grid, FB_THREADS, 0, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace moe
