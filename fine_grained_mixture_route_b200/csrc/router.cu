// CUDA-core router of the DeepSeekMoE layer ("《DeepSeekMoE》深度解读报告" §3.1, Eq. 3-5 in
// prose): z = x . e_i for every expert centroid, softmax over all N_m experts, keep the
// N_r largest probabilities as gates (no renormalisation; ties to the lower index).  Also the
// two router variants: softmax over the top-k logits of a biased router (the FineGrainedMoE
// listing of the DeepSeek-V2 explainer, §3.1) and a sigmoid gate with a selection-only bias.
//
// Used for fp32 layers and for expert counts the tensor-core router does not take.  Phase
// 1 computes a [32 tokens x N_m] block of fp32 logits from shared-memory tiles of x and the
// centroids; phase 2 gives each token to one warp, which keeps the token's logits in shared
// memory, reduces max and sum-of-exponentials with shuffles and takes N_r rounds of warp
// argmax on the key (logit, -index).
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int RT_TOK = 32;      // tokens per block
constexpr int RT_EXP = 64;      // experts per score tile
constexpr int RT_K = 64;        // hidden elements per score tile
constexpr int RT_THREADS = 256;

// Picks and gates of one token by one warp from its E logits zr (shared memory, unchanged).
// The selection key is z + bias (gate modes 0 and 1) or sigmoid(z) + bias (mode 2); lane l owns
// experts l + 32 i and marks its picks in a bit mask.  k rounds of warp argmax on (key, -index)
// give the picks in descending key, equal keys to the lower index.  Gates: mode 0 the softmax of
// z + bias over all E experts read at the picks; mode 1 the softmax over the k picked keys;
// mode 2 sigmoid(z) at the picks divided by their sum.
__device__ void warp_route(const float* zr, int E, int k, int mode, const float* __restrict__ bias, int lane,
                           int32_t* idx_row, float* gate_row) {
    auto key_of = [&](int e) {
        const float z = zr[e];
        const float bb = bias ? bias[e] : 0.f;
        return mode == 2 ? 1.0f / (1.0f + expf(-z)) + bb : z + bb;
    };
    float m = -INFINITY, inv = 0.f;
    if (mode == 0) {
        for (int e = lane; e < E; e += 32) m = fmaxf(m, key_of(e));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float s = 0.f;
        for (int e = lane; e < E; e += 32) s += expf(key_of(e) - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        inv = 1.0f / s;
    }
    uint32_t taken = 0;
    float first = 0.f, norm = 0.f;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int e = lane, i = 0; e < E; e += 32, ++i) {
            if (taken & (1u << i)) continue;
            const float v = key_of(e);
            if (v > bv) { bv = v; bi = e; }     // ascending e: equal keys keep the lower index
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (bi < E && (bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == 0) {
            idx_row[j] = bi;
            float g;
            if (mode == 0) {
                g = expf(bv - m) * inv;
            } else if (mode == 1) {
                if (j == 0) first = bv;
                g = expf(bv - first);
                norm += g;
            } else {
                g = 1.0f / (1.0f + expf(-zr[bi]));
                norm += g;
            }
            gate_row[j] = g;
        }
        __syncwarp();
    }
    if (lane == 0 && mode != 0) {
        const float r = 1.0f / norm;
        for (int j = 0; j < k; ++j) gate_row[j] *= r;
    }
}

template <typename T>
__global__ void __launch_bounds__(RT_THREADS)
router_simt_kernel(const T* __restrict__ x, const T* __restrict__ cen, const float* __restrict__ bias, int mode,
                   int32_t* __restrict__ idx_out, float* __restrict__ gate_out, int Tn, int d, int E, int k) {
    extern __shared__ float sm[];
    float* xs = sm;                                  // [RT_TOK][RT_K + 1]
    float* cs = xs + RT_TOK * (RT_K + 1);            // [RT_EXP][RT_K + 1]
    float* z = cs + RT_EXP * (RT_K + 1);             // [RT_TOK][E]
    const int t0 = blockIdx.x * RT_TOK;
    const int tid = threadIdx.x;
    const int tt = tid / 8;                          // token of this thread in phase 1
    const int eo = tid % 8;                          // expert lane: experts eo + 8q

    for (int e0 = 0; e0 < E; e0 += RT_EXP) {
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int k0 = 0; k0 < d; k0 += RT_K) {
            __syncthreads();
            for (int i = tid; i < RT_TOK * RT_K; i += RT_THREADS) {
                int r = i / RT_K, c = i % RT_K;
                int t = t0 + r, kk = k0 + c;
                xs[r * (RT_K + 1) + c] = (t < Tn && kk < d) ? to_f32(x[(size_t)t * d + kk]) : 0.f;
            }
            for (int i = tid; i < RT_EXP * RT_K; i += RT_THREADS) {
                int r = i / RT_K, c = i % RT_K;
                int e = e0 + r, kk = k0 + c;
                cs[r * (RT_K + 1) + c] = (e < E && kk < d) ? to_f32(cen[(size_t)e * d + kk]) : 0.f;
            }
            __syncthreads();
#pragma unroll 4
            for (int c = 0; c < RT_K; ++c) {
                float xv = xs[tt * (RT_K + 1) + c];
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = fmaf(xv, cs[(eo + 8 * q) * (RT_K + 1) + c], acc[q]);
            }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            int e = e0 + eo + 8 * q;
            if (e < E) z[tt * E + e] = acc[q];
        }
    }
    __syncthreads();

    // phase 2: one warp per token
    const int warp = tid / 32, lane = tid % 32;
    for (int r = warp; r < RT_TOK; r += RT_THREADS / 32) {
        const int t = t0 + r;
        if (t >= Tn) break;
        warp_route(z + r * E, E, k, mode, bias, lane, idx_out + (size_t)t * k, gate_out + (size_t)t * k);
    }
}


// Split-K router, last step: z = sum of the per-split partial logits in ascending split order
// (deterministic), then the same softmax / top-k as above.  One block per token: E/4 threads
// each sum a float4 of consecutive experts over the splits (coalesced across the block), then
// warp 0 ranks the token.
__global__ void __launch_bounds__(256)
router_finish_kernel(const float* __restrict__ partial, int nsplit, int Tn, int E, int k, const float* __restrict__ bias,
                     int mode, int32_t* __restrict__ idx_out, float* __restrict__ gate_out) {
    extern __shared__ float zs[];
    const int t = blockIdx.x;
    const int E4 = E / 4;
    const size_t stride4 = (size_t)Tn * E4;                 // float4s between consecutive splits
    for (int e4 = threadIdx.x; e4 < E4; e4 += blockDim.x) {
        const float4* src = reinterpret_cast<const float4*>(partial) + (size_t)t * E4 + e4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        int s = 0;
        for (; s + 4 <= nsplit; s += 4) {
            const float4 v0 = src[(size_t)s * stride4], v1 = src[(size_t)(s + 1) * stride4];
            const float4 v2 = src[(size_t)(s + 2) * stride4], v3 = src[(size_t)(s + 3) * stride4];
            acc.x += v0.x; acc.y += v0.y; acc.z += v0.z; acc.w += v0.w;
            acc.x += v1.x; acc.y += v1.y; acc.z += v1.z; acc.w += v1.w;
            acc.x += v2.x; acc.y += v2.y; acc.z += v2.z; acc.w += v2.w;
            acc.x += v3.x; acc.y += v3.y; acc.z += v3.z; acc.w += v3.w;
        }
        for (; s < nsplit; ++s) {
            const float4 v = src[(size_t)s * stride4];
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        reinterpret_cast<float4*>(zs)[e4] = acc;
    }
    __syncthreads();
    if (threadIdx.x < 32) warp_route(zs, E, k, mode, bias, threadIdx.x, idx_out + (size_t)t * k, gate_out + (size_t)t * k);
}

}  // namespace

cudaError_t launch_router_simt(const Dims& D, const void* x, const void* centroids, const float* bias, int32_t* idx,
                               float* gate, cudaStream_t stream) {
    const int blocks = ceil_div(D.T, RT_TOK);
    const size_t smem = sizeof(float) * ((size_t)RT_TOK * (RT_K + 1) + (size_t)RT_EXP * (RT_K + 1) + (size_t)RT_TOK * D.E);
    if (D.bf16) {
        auto kern = router_simt_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<blocks, RT_THREADS, smem, stream>>>((const __nv_bfloat16*)x, (const __nv_bfloat16*)centroids, bias,
                                                   D.gate_mode, idx, gate, D.T, D.d, D.E, D.k);
    } else {
        auto kern = router_simt_kernel<float>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<blocks, RT_THREADS, smem, stream>>>((const float*)x, (const float*)centroids, bias, D.gate_mode, idx, gate,
                                                   D.T, D.d, D.E, D.k);
    }
    return cudaGetLastError();
}

cudaError_t launch_router_finish(const Dims& D, const float* partial, int nsplit, const float* bias, int32_t* idx,
                                 float* gate, cudaStream_t stream) {
    const int E4 = D.E / 4;
    const int threads = E4 < 32 ? 32 : (E4 > 256 ? 256 : (E4 + 31) / 32 * 32);
    router_finish_kernel<<<D.T, threads, sizeof(float) * D.E, stream>>>(partial, nsplit, D.T, D.E, D.k, bias,
                                                                         D.gate_mode, idx, gate);
    return cudaGetLastError();
}

}  // namespace moe
