// Backward pass of the layer: the kernels around the tensor-core GEMMs (tile tables of the
// padded groups, row gathers, the router's backward, bias-gradient column sums).
//
// Chain rule of the forward (per routed slot p = (t, j) of expert e, gate g_p):
//   dy_p = g_p dout_t;  dgate_p = <dout_t, y_p> = <dout_t W2_e, h_p> + <dout_t, b2_e>
//   dh_p = g_p (dout_t W2_e);  da = dh g_pre sigmoid'(a)-term;  dg = dh silu(a)      (DH GEMM epilogue)
//   dx_t += da W1_e + dg W3_e (DX GEMM)  + shared experts + dz_t C (DXS GEMM)
//   dW2_e = sum_p dy_p h_p^T, dW1_e = sum_p da_p x_t^T, dW3_e = sum_p dg_p x_t^T   (DW GEMMs)
//   dz_t from dgate_t by the gate mode's softmax / sigmoid backward (router_bwd_kernel).
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

__device__ __forceinline__ int round64(int n) { return (n + 63) & ~63; }

// inclusive scan of v over the block (blockDim.x <= 1024, a multiple of 32)
__device__ int block_inclusive_scan(int v, int* warp_sums) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) warp_sums[w] = v;
    __syncthreads();
    if (w == 0) {
        int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += n;
        }
        if (lane < nw) warp_sums[lane] = s;
    }
    __syncthreads();
    const int r = v + (w > 0 ? warp_sums[w - 1] : 0);
    __syncthreads();
    return r;
}

// offs_pad[e] = sum_{e' < e} round64(count_e'); ts_dh over routed + shared groups (128-row x 256-col
// tiles of the DH GEMM), ts_dx over routed groups (DX GEMM).  One block of 1024 threads, looping
// over chunks of 1024 experts.
__global__ void __launch_bounds__(1024) plan_bwd_kernel(const int32_t* __restrict__ offsets, int E, int Ks, int T, int d,
                                                        int I, int Is, int32_t* offs_pad, int32_t* ts_dh,
                                                        int32_t* ts_dx) {
    __shared__ int ws[32];
    __shared__ int carry[3];
    if (threadIdx.x == 0) { carry[0] = carry[1] = carry[2] = 0; offs_pad[0] = 0; ts_dh[0] = 0; ts_dx[0] = 0; }
    __syncthreads();
    const int G = E + Ks;
    for (int base = 0; base < G; base += blockDim.x) {
        const int g = base + threadIdx.x;
        int cpad = 0, tdh = 0, tdx = 0;
        if (g < E) {
            const int c = offsets[g + 1] - offsets[g];
            cpad = round64(c);
            tdh = ceil_div(c, 128) * ceil_div(I, 256);
            tdx = ceil_div(c, 128) * ceil_div(d, 256);
        } else if (g < G) {
            tdh = ceil_div(T, 128) * ceil_div(Is, 256);
        }
        const int s0 = block_inclusive_scan(cpad, ws);
        const int s1 = block_inclusive_scan(tdh, ws);
        const int s2 = block_inclusive_scan(tdx, ws);
        if (g < E) { offs_pad[g + 1] = carry[0] + s0; ts_dx[g + 1] = carry[2] + s2; }
        if (g < G) ts_dh[g + 1] = carry[1] + s1;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) { carry[0] += s0; carry[1] += s1; carry[2] += s2; }
        __syncthreads();
    }
}

__device__ __forceinline__ int group_of(const int32_t* starts, int n, int q) {   // largest g with starts[g] <= q
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (starts[mid] <= q) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Rows of the padded grouped layout: q in [0, offs_pad[E]).  A live row (slot p = offsets[e] + r)
// gets dout and x of its token, its gate, and b2dot[p] = <dout_t, b2_e>; a pad row gets zeros.
// x_pad rows end with 64 extra columns (1 for a live row, then zeros) and hg rows (I + 64 long,
// whose first I columns the DH GEMM writes) with the gate, then zeros.
__global__ void bwd_gather_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ x,
                                  const __nv_bfloat16* __restrict__ b2, const int32_t* __restrict__ offsets,
                                  const int32_t* __restrict__ offs_pad, const int32_t* __restrict__ stok,
                                  const float* __restrict__ sgate, int E, int T, int d, int I, uint4* dout_pad,
                                  uint4* x_pad, __nv_bfloat16* hg, float* gate_pad, float* b2dot, uint32_t* err) {
    __shared__ float red[32];
    const int nv = d / 8;
    const int nvx = nv + 8;                         // x_pad row: d + 64 bf16
    const int total = offs_pad[E];
    for (int q = blockIdx.x; q < total; q += gridDim.x) {
        const int e = group_of(offs_pad, E, q);
        const int r = q - offs_pad[e];
        const bool live = r < offsets[e + 1] - offsets[e];
        const int p = offsets[e] + r;
        int t = live ? stok[p] : -1;
        if (live && (t < 0 || t >= T)) {
            if (threadIdx.x == 0) flag_error(err, ERR_INDEX_RANGE);
            t = -1;
        }
        float dot = 0.f;
        for (int i = threadIdx.x; i < nv; i += blockDim.x) {
            uint4 dv = make_uint4(0, 0, 0, 0), xv = make_uint4(0, 0, 0, 0);
            if (t >= 0) {
                dv = __ldg(dout + (size_t)t * nv + i);
                xv = __ldg(x + (size_t)t * nv + i);
                if (b2) {
                    const uint4 bv = *reinterpret_cast<const uint4*>(b2 + (size_t)e * d + i * 8);
                    const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        dot += __uint_as_float(dw[k] << 16) * __uint_as_float(bw[k] << 16) +
                               __uint_as_float(dw[k] & 0xFFFF0000u) * __uint_as_float(bw[k] & 0xFFFF0000u);
                }
            }
            dout_pad[(size_t)q * nv + i] = dv;
            x_pad[(size_t)q * nvx + i] = xv;
        }
        const float gq = t >= 0 ? sgate[p] : 0.f;
        if (threadIdx.x < 8) {
            const uint32_t one = t >= 0 ? 0x3F80u : 0u;                     // bf16 1.0
            const uint32_t gb = __bfloat16_as_ushort(__float2bfloat16_rn(gq));
            x_pad[(size_t)q * nvx + nv + threadIdx.x] = make_uint4(threadIdx.x == 0 ? one : 0u, 0, 0, 0);
            reinterpret_cast<uint4*>(hg + (size_t)q * (I + 64) + I)[threadIdx.x] =
                make_uint4(threadIdx.x == 0 ? gb : 0u, 0, 0, 0);
        }
        if (threadIdx.x == 0) gate_pad[q] = gq;
        if (b2 && live) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            __syncthreads();
            if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = dot;
            __syncthreads();
            if (threadIdx.x == 0) {
                float s = 0.f;
                for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
                b2dot[p] = s;
            }
        }
    }
}

// One warp per token: dgate_j = sum of the DH partials of its slot (+ <dout, b2>), then the gate
// mode's backward to the logits, dz [T][N_m] in fp32 and bf16 (the A operand of dz . C and dz^T x).
__global__ void router_bwd_kernel(const float* __restrict__ z, const float* __restrict__ bias,
                                  const int32_t* __restrict__ idx, const int32_t* __restrict__ slot_of,
                                  const float* __restrict__ dgate_part, int n_parts, const float* __restrict__ b2dot,
                                  int T, int E, int k, int mode, float* dz, __nv_bfloat16* dz_bf16, float* dgate_out) {
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
        // gate gradients of the k picks (lane j holds pick j)
        float dgj = 0.f;
        int ij = -1;
        if (lane < k) {
            const int p = slot_of[(size_t)t * k + lane];
            ij = idx[(size_t)t * k + lane];
            if (ij < 0 || ij >= E || p < 0 || p >= T * k) {      // picks come from the forward; guard anyway
                ij = 0;
            } else {
                for (int q = 0; q < n_parts; ++q) dgj += dgate_part[(size_t)p * n_parts + q];
                if (b2dot) dgj += b2dot[p];
            }
            if (dgate_out) dgate_out[(size_t)t * k + lane] = dgj;
        }
        const float* zr = z + (size_t)t * E;
        float* dzr = dz + (size_t)t * E;
        __nv_bfloat16* dzb = dz_bf16 + (size_t)t * E;
        if (mode == 0) {
            // s = softmax(z + bias); dz_i = [i picked] dgate_j s_i - s_i sum_j dgate_j s_{idx_j}
            float m = -INFINITY;
            for (int i = lane; i < E; i += 32) m = fmaxf(m, zr[i] + (bias ? bias[i] : 0.f));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            float sum = 0.f;
            for (int i = lane; i < E; i += 32) sum += expf(zr[i] + (bias ? bias[i] : 0.f) - m);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            const float sj = lane < k ? expf(zr[ij] + (bias ? bias[ij] : 0.f) - m) / sum : 0.f;
            float wsum = sj * dgj;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
            for (int i = lane; i < E; i += 32) {
                const float si = expf(zr[i] + (bias ? bias[i] : 0.f) - m) / sum;
                float v = -si * wsum;
                for (int j = 0; j < k; ++j) {
                    const int ii = __shfl_sync(0xffffffffu, ij, j);
                    const float dd = __shfl_sync(0xffffffffu, dgj, j);
                    if (ii == i) v += dd * si;
                }
                dzr[i] = v;
                dzb[i] = __float2bfloat16_rn(v);
            }
        } else {
            // modes 1 and 2: the gradient lives on the picks only
            float gj = 0.f, sgj = 0.f;
            if (lane < k) {
                const float zj = zr[ij] + ((mode == 1 && bias) ? bias[ij] : 0.f);
                gj = zj;
                if (mode == 2) sgj = 1.0f / (1.0f + expf(-zr[ij]));
            }
            float tot;
            if (mode == 1) {
                float m = lane < k ? gj : -INFINITY;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                const float ev = lane < k ? expf(gj - m) : 0.f;
                tot = ev;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
                gj = ev / tot;                                       // the gate of pick j
            } else {
                tot = sgj;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
                gj = lane < k ? sgj / tot : 0.f;
            }
            float gd = gj * dgj;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) gd += __shfl_xor_sync(0xffffffffu, gd, o);
            float dj = 0.f;
            if (lane < k) dj = mode == 1 ? gj * (dgj - gd) : sgj * (1.0f - sgj) * (dgj - gd) / tot;
            for (int i = lane; i < E; i += 32) {
                float v = 0.f;
                for (int j = 0; j < k; ++j) {
                    const int ii = __shfl_sync(0xffffffffu, ij, j);
                    const float dd = __shfl_sync(0xffffffffu, dj, j);
                    if (ii == i) v += dd;
                }
                dzr[i] = v;
                dzb[i] = __float2bfloat16_rn(v);
            }
        }
    }
}

// Column sums over the T rows of each group, deterministic, in two passes:
//   partial[g][j][c] = sum of rows [256 j, 256 j + 256) of src_g[.][c]  (src_g = src + g * group_stride)
//   out[g][c] = sum_j partial[g][j][c] in order; columns c < split -> out0[g][c], the rest -> out1[g][c - split]
constexpr int COLSUM_ROWS = 256;
template <typename TS>
__global__ void colsum_partial_kernel(const TS* __restrict__ src, long long group_stride, int ld, int n_rows, int W,
                                      float* partial) {
    const int g = blockIdx.z, j = blockIdx.y;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= W) return;
    const int nch = (n_rows + COLSUM_ROWS - 1) / COLSUM_ROWS;
    const TS* base = src + (size_t)g * group_stride;
    const int r0 = j * COLSUM_ROWS, r1 = min(n_rows, r0 + COLSUM_ROWS);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int r = r0;
    for (; r + 3 < r1; r += 4) {
        a0 += to_f32<TS>(base[(size_t)r * ld + c]);
        a1 += to_f32<TS>(base[(size_t)(r + 1) * ld + c]);
        a2 += to_f32<TS>(base[(size_t)(r + 2) * ld + c]);
        a3 += to_f32<TS>(base[(size_t)(r + 3) * ld + c]);
    }
    for (; r < r1; ++r) a0 += to_f32<TS>(base[(size_t)r * ld + c]);
    partial[((size_t)g * nch + j) * W + c] = (a0 + a1) + (a2 + a3);
}

template <typename TO>
__global__ void colsum_final_kernel(const float* __restrict__ partial, int nch, int W, int split, TO* out0, TO* out1) {
    const int g = blockIdx.y;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= W) return;
    float acc = 0.f;
    for (int j = 0; j < nch; ++j) acc += partial[((size_t)g * nch + j) * W + c];
    if (c < split) out0[(size_t)g * split + c] = from_f32<TO>(acc);
    else out1[(size_t)g * (W - split) + (c - split)] = from_f32<TO>(acc);
}

// hg_s rows (K_s x T, I_s + 64 long): column I_s = 1, the other extra columns 0
__global__ void fill_aug_kernel(__nv_bfloat16* rows, long long n_rows, int ld, int col) {
    const long long n = n_rows * 8;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const long long r = i / 8;
        const int j = (int)(i % 8);
        reinterpret_cast<uint4*>(rows + (size_t)r * ld + col)[j] = make_uint4(j == 0 ? 0x3F80u : 0u, 0, 0, 0);
    }
}

// One warp per token: the row of router logits z (fp32, in place) becomes the score
// distribution the balance statistics average: softmax of z + bias (gate modes 0, 1) or
// sigmoid(z) normalised over the experts (mode 2).
__global__ void balance_scores_kernel(float* z, const float* __restrict__ bias, int T, int E, int mode) {
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
        float* zr = z + (size_t)t * E;
        if (mode == 2) {
            float sum = 0.f;
            for (int i = lane; i < E; i += 32) sum += 1.0f / (1.0f + expf(-zr[i]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            __syncwarp();
            for (int i = lane; i < E; i += 32) zr[i] = (1.0f / (1.0f + expf(-zr[i]))) / sum;
        } else {
            float m = -INFINITY;
            for (int i = lane; i < E; i += 32) m = fmaxf(m, zr[i] + (bias ? bias[i] : 0.f));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            float sum = 0.f;
            for (int i = lane; i < E; i += 32) sum += expf(zr[i] + (bias ? bias[i] : 0.f) - m);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            __syncwarp();
            for (int i = lane; i < E; i += 32) zr[i] = expf(zr[i] + (bias ? bias[i] : 0.f) - m) / sum;
        }
    }
}

// f_i = N_m / (N_r T) * counts_i, P_i = Psum_i / T, terms[0] = sum_i f_i P_i, terms[1] = sum over
// n_groups equal contiguous groups of mean(f) * sum(P).  One block, fixed summation order.
__global__ void balance_final_kernel(const float* __restrict__ psum, const int32_t* __restrict__ counts, int T, int E,
                                     int k, int n_groups, float* f, float* P, float* terms) {
    __shared__ float fs[1024], ps[1024];
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
        const float fi = (float)counts[i] * (float)E / ((float)k * (float)T);
        const float pi = psum[i] / (float)T;
        f[i] = fi; P[i] = pi; fs[i] = fi; ps[i] = pi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float te = 0.f, td = 0.f;
        for (int i = 0; i < E; ++i) te += fs[i] * ps[i];
        const int per = E / n_groups;
        for (int g = 0; g < n_groups; ++g) {
            float fg = 0.f, pg = 0.f;
            for (int i = g * per; i < (g + 1) * per; ++i) { fg += fs[i]; pg += ps[i]; }
            td += (fg / (float)per) * pg;
        }
        terms[0] = te;
        terms[1] = td;
    }
}

}  // namespace

cudaError_t launch_balance(const Dims& D, float* z, const float* bias, const int32_t* counts, int n_groups,
                           float* partial, float* psum, float* f, float* P, float* terms, cudaStream_t stream) {
    if (D.T == 0) return cudaSuccess;
    const long long need = (D.T + 7) / 8, cap = (long long)num_sms() * 8;
    balance_scores_kernel<<<(int)(need < cap ? need : cap), 256, 0, stream>>>(
        z, D.gate_mode == MOE_GATE_SIGMOID_BIAS ? nullptr : bias, D.T, D.E, D.gate_mode);
    cudaError_t e = launch_colsum(true, true, z, 0, D.E, D.T, 1, D.E, D.E, psum, nullptr, partial, stream);
    if (e != cudaSuccess) return e;
    balance_final_kernel<<<1, 256, 0, stream>>>(psum, counts, D.T, D.E, D.k, n_groups, f, P, terms);
    return cudaGetLastError();
}

cudaError_t launch_plan_bwd(const Dims& D, const int32_t* offsets, int32_t* offs_pad, int32_t* ts_dh, int32_t* ts_dx,
                            cudaStream_t stream) {
    plan_bwd_kernel<<<1, 1024, 0, stream>>>(offsets, D.E, D.Ks, D.T, D.d, D.I, D.Ks ? D.Is : 0, offs_pad, ts_dh, ts_dx);
    return cudaGetLastError();
}

cudaError_t launch_bwd_gather(const Dims& D, const void* dout, const void* x, const void* b2, const int32_t* offsets,
                              const int32_t* offs_pad, const int32_t* stok, const float* sgate, void* dout_pad,
                              void* x_pad, void* hg, float* gate_pad, float* b2dot, uint32_t* err, cudaStream_t stream) {
    if (D.T == 0) return cudaSuccess;
    const long long rows = D.slots() + 64LL * D.E;
    const long long cap = (long long)num_sms() * 16;
    bwd_gather_kernel<<<(int)(rows < cap ? rows : cap), 128, 0, stream>>>(
        (const uint4*)dout, (const uint4*)x, (const __nv_bfloat16*)b2, offsets, offs_pad, stok, sgate, D.E, D.T, D.d, D.I,
        (uint4*)dout_pad, (uint4*)x_pad, (__nv_bfloat16*)hg, gate_pad, b2dot, err);
    return cudaGetLastError();
}

cudaError_t launch_router_bwd(const Dims& D, const float* z, const float* bias, const int32_t* idx,
                              const int32_t* slot_of, const float* dgate_part, int n_parts, const float* b2dot,
                              float* dz, void* dz_bf16, float* dgate_out, cudaStream_t stream) {
    if (D.T == 0) return cudaSuccess;
    const int warps = 8;
    const long long need = (D.T + warps - 1) / warps;
    const long long cap = (long long)num_sms() * 8;
    router_bwd_kernel<<<(int)(need < cap ? need : cap), warps * 32, 0, stream>>>(
        z, D.gate_mode == MOE_GATE_SIGMOID_BIAS ? nullptr : bias, idx, slot_of, dgate_part, n_parts, b2dot, D.T, D.E,
        D.k, D.gate_mode, dz, (__nv_bfloat16*)dz_bf16, dgate_out);
    return cudaGetLastError();
}

cudaError_t launch_colsum(bool src_f32, bool out_f32, const void* src, long long group_stride, int ld, int n_rows,
                          int groups, int W, int split, void* out0, void* out1, float* partial, cudaStream_t stream) {
    if (groups <= 0 || W <= 0 || n_rows <= 0) return cudaSuccess;
    if (!out1) split = W;
    const int nch = (n_rows + COLSUM_ROWS - 1) / COLSUM_ROWS;
    const dim3 g1((W + 255) / 256, nch, groups), g2((W + 255) / 256, groups);
    if (src_f32) colsum_partial_kernel<float><<<g1, 256, 0, stream>>>((const float*)src, group_stride, ld, n_rows, W, partial);
    else colsum_partial_kernel<__nv_bfloat16><<<g1, 256, 0, stream>>>((const __nv_bfloat16*)src, group_stride, ld,
                                                                      n_rows, W, partial);
    if (out_f32) colsum_final_kernel<float><<<g2, 256, 0, stream>>>(partial, nch, W, split, (float*)out0, (float*)out1);
    else colsum_final_kernel<__nv_bfloat16><<<g2, 256, 0, stream>>>(partial, nch, W, split, (__nv_bfloat16*)out0,
                                                                    (__nv_bfloat16*)out1);
    return cudaGetLastError();
}

cudaError_t launch_fill_aug(void* rows, long long n_rows, int ld, int col, cudaStream_t stream) {
    if (n_rows <= 0) return cudaSuccess;
    const long long n = n_rows * 8;
    const long long cap = (long long)num_sms() * 8;
    const long long blocks = (n + 255) / 256;
    fill_aug_kernel<<<(int)(blocks < cap ? blocks : cap), 256, 0, stream>>>((__nv_bfloat16*)rows, n_rows, ld, col);
    return cudaGetLastError();
}

}  // namespace moe
