// Per-expert token lists, the grouped GEMMs' tile tables, the row gather and the combine.
//
// The grouping follows the "top-k indices first, then gather the tokens of each expert"
// step of the DeepSeek-V2 explainer (eliteato.com/news/32734, §3.1 and §3.3): the T*N_r
// slots (slot s = t*N_r + j) are grouped by expert in three passes — a per-block histogram,
// a scan over (expert, block), and a scatter that ranks equal experts inside a warp with
// __match_any_sync.  Inside an expert the slots keep ascending order, so the result does not
// depend on scheduling (no order-dependent atomics).
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int SCAN_THREADS = 1024;

// Exclusive scan of n values in place by one block; returns the total.  Each thread owns a
// contiguous run of ceil(n / blockDim) values; run sums are scanned with warp shuffles.
__device__ int block_exclusive_scan(int* v, int n, int* warp_sums) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (n + nt - 1) / nt;
    const int b = tid * per, e = min(n, b + per);
    int run = 0;
    for (int i = b; i < e; ++i) run += v[i];
    // inclusive warp scan of run
    int incl = run;
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int nw = nt / 32;
        int ws = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, ws, o);
            if (lane >= o) ws += y;
        }
        if (lane < nw) warp_sums[lane] = ws;   // inclusive warp prefix
    }
    __syncthreads();
    int base = (warp > 0 ? warp_sums[warp - 1] : 0) + incl - run;
    const int total = warp_sums[nt / 32 - 1];
    for (int i = b; i < e; ++i) {
        int t = v[i];
        v[i] = base;
        base += t;
    }
    __syncthreads();
    return total;
}

// pass 1: per-block histogram of expert picks
__global__ void permute_hist_kernel(const int32_t* __restrict__ idx, long long S, int E,
                                    int32_t* __restrict__ block_hist, uint32_t* err) {
    extern __shared__ int hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const long long s0 = (long long)blockIdx.x * PERMUTE_CHUNK;
    const long long s1 = min(S, s0 + PERMUTE_CHUNK);
    for (long long s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
        int e = idx[s];
        if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
        else flag_error(err, ERR_EXPERT_RANGE);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) block_hist[(size_t)blockIdx.x * E + e] = hist[e];
}

// pass 2: counts, offsets, and each block's starting position per expert (in place).  One
// thread per expert walks that expert's column of block counts (consecutive threads read
// consecutive experts of a block row, so every load is coalesced; loads are unrolled).
__global__ void permute_scan_kernel(int32_t* __restrict__ block_hist, int nblk, int E,
                                    int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
    extern __shared__ int sh[];
    int* cnt = sh;               // [E]
    int* warp_sums = sh + E;     // [32]
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        int b = 0;
        for (; b + 8 <= nblk; b += 8) {
            int c[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) c[i] = block_hist[(size_t)(b + i) * E + e];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                block_hist[(size_t)(b + i) * E + e] = run;
                run += c[i];
            }
        }
        for (; b < nblk; ++b) {
            const int c = block_hist[(size_t)b * E + e];
            block_hist[(size_t)b * E + e] = run;
            run += c;
        }
        cnt[e] = run;
        counts[e] = run;
    }
    __syncthreads();
    const int total = block_exclusive_scan(cnt, E, warp_sums);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        offsets[e] = cnt[e];
        const int base = cnt[e];
        for (int b = 0; b < nblk; ++b) block_hist[(size_t)b * E + e] += base;
    }
    if (threadIdx.x == 0) offsets[E] = total;
}

// pass 3: one warp per block walks its chunk of slots in order, 32 at a time.  The chunk's
// picks and gates are loaded up front (32 per lane), so the ordered walk itself only touches
// shared memory and issues independent stores.
__global__ void __launch_bounds__(32) permute_scatter_kernel(const int32_t* __restrict__ idx,
                                                             const float* __restrict__ gate, long long S, int k,
                                                             int E, const int32_t* __restrict__ block_base,
                                                             int32_t* __restrict__ sorted_token,
                                                             float* __restrict__ sorted_gate,
                                                             int32_t* __restrict__ slot_of) {
    constexpr int STEPS = PERMUTE_CHUNK / 32;
    extern __shared__ int running[];
    const int lane = threadIdx.x;
    for (int e = lane; e < E; e += 32) running[e] = block_base[(size_t)blockIdx.x * E + e];
    const long long s0 = (long long)blockIdx.x * PERMUTE_CHUNK;
    const long long s1 = min(S, s0 + PERMUTE_CHUNK);
    int ev[STEPS];
    float gv[STEPS];
#pragma unroll
    for (int i = 0; i < STEPS; ++i) {
        const long long s = s0 + 32 * i + lane;
        ev[i] = s < s1 ? idx[s] : -1;
        gv[i] = s < s1 ? gate[s] : 0.f;
    }
    __syncwarp();
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < STEPS; ++i) {
        const long long s = s0 + 32 * i + lane;
        if (s0 + 32 * i >= s1) break;
        const bool live = s < s1;
        int e = ev[i];
        const bool ok = live && e >= 0 && e < E;
        if (!ok) e = -1 - lane;                       // unique key: never matches a real expert
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        int pos = 0;
        if (ok) pos = running[e] + __popc(peers & lt);
        __syncwarp();
        if (ok && (peers & lt) == 0) running[e] += __popc(peers);   // group leader advances
        __syncwarp();
        if (ok) {
            sorted_token[pos] = (int32_t)(s / k);
            sorted_gate[pos] = gv[i];
            slot_of[s] = pos;
        } else if (live) {
            slot_of[s] = -1;
        }
    }
}

// The three passes in one block for small groupings (PERMUTE_SMALL_SLOTS slots at most, at most
// PERMUTE_SMALL_EXPERTS experts): its 32 warps play the part of the histogram / scatter blocks, warp w
// taking the w-th consecutive slice of the slots, so the order inside an expert is again ascending
// slot order and the result equals the multi-block passes' bit for bit.  Shared memory: a histogram
// row per warp [32][E], then the expert totals [E] and 32 scan partials.
__global__ void __launch_bounds__(1024) permute_small_kernel(const int32_t* __restrict__ idx,
                                                             const float* __restrict__ gate, long long S, int k, int E,
                                                             int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ sorted_token,
                                                             float* __restrict__ sorted_gate,
                                                             int32_t* __restrict__ slot_of, uint32_t* err) {
    extern __shared__ int sh[];
    int* hist = sh;                   // [32][E]: counts, then each warp's running position per expert
    int* cnt = sh + 32 * E;           // [E]
    int* wsum = cnt + E;              // [32]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long chunk = (S + 31) / 32;
    const long long s0 = warp * chunk, s1 = min(S, s0 + chunk);
    for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (long long s = s0 + lane; s < s1; s += 32) {
        const int e = idx[s];
        if (e >= 0 && e < E) atomicAdd(&hist[warp * E + e], 1);
        else flag_error(err, ERR_EXPERT_RANGE);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {         // warp-order bases inside each expert
        int run = 0;
        for (int w = 0; w < 32; ++w) {
            const int c = hist[w * E + e];
            hist[w * E + e] = run;
            run += c;
        }
        cnt[e] = run;
        counts[e] = run;
    }
    __syncthreads();
    const int total = block_exclusive_scan(cnt, E, wsum);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        offsets[e] = cnt[e];
        for (int w = 0; w < 32; ++w) hist[w * E + e] += cnt[e];
    }
    if (threadIdx.x == 0) offsets[E] = total;
    __syncthreads();
    int* running = hist + warp * E;
    const unsigned lt = (1u << lane) - 1u;
    for (long long b = s0; b < s1; b += 32) {
        const long long s = b + lane;
        const bool live = s < s1;
        int e = live ? idx[s] : -1;
        const float g = live ? gate[s] : 0.f;
        const bool ok = live && e >= 0 && e < E;
        if (!ok) e = -1 - lane;                       // unique key: never matches a real expert
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        int pos = 0;
        if (ok) pos = running[e] + __popc(peers & lt);
        __syncwarp();
        if (ok && (peers & lt) == 0) running[e] += __popc(peers);   // group leader advances
        __syncwarp();
        if (ok) {
            sorted_token[pos] = (int32_t)(s / k);
            sorted_gate[pos] = g;
            slot_of[s] = pos;
        } else if (live) {
            slot_of[s] = -1;
        }
    }
}

// tile tables of the grouped GEMMs (see launch.h)
__global__ void plan_kernel(const int32_t* __restrict__ offsets, long long S, int T, int d, int E, int I, int Ks,
                            int Is, int tile_rows, int32_t* __restrict__ tile_start1, int32_t* __restrict__ tile_start2, uint32_t* err) {
    extern __shared__ int sh[];
    const int G = E + Ks;
    int* t1 = sh;                // [G + 1]
    int* t2 = sh + G + 1;        // [E + 1]
    int* warp_sums = t2 + E + 1; // [32]
    const int n1r = ceil_div(I, 128), n1s = ceil_div(Is, 128), n2 = ceil_div(d, 256);
    // caller-supplied offsets must be a grouping of the T*k slots: offsets[0] = 0,
    // non-decreasing, offsets[E] = T*k.  Otherwise no routed tile is planned at all.
    __shared__ int bad;
    if (threadIdx.x == 0) bad = offsets ? (offsets[0] != 0 || (long long)offsets[E] != S) : 0;
    __syncthreads();
    if (offsets)
        for (int g = threadIdx.x; g < E; g += blockDim.x)
            if (offsets[g + 1] < offsets[g]) bad = 1;
    __syncthreads();
    if (bad && threadIdx.x == 0) flag_error(err, ERR_INDEX_RANGE);
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        int rows;
        if (g < E) {
            rows = (offsets && !bad) ? offsets[g + 1] - offsets[g] : 0;
        } else {
            rows = T;
        }
        const int m = ceil_div(rows, tile_rows);
        t1[g] = m * (g < E ? n1r : n1s);
        if (g < E) t2[g] = m * n2;
    }
    __syncthreads();
    const int tot1 = block_exclusive_scan(t1, G, warp_sums);
    const int tot2 = block_exclusive_scan(t2, E, warp_sums);
    for (int g = threadIdx.x; g < G; g += blockDim.x) tile_start1[g] = t1[g];
    for (int e = threadIdx.x; e < E; e += blockDim.x) tile_start2[e] = t2[e];
    if (threadIdx.x == 0) {
        tile_start1[G] = tot1;
        tile_start2[E] = tot2;
    }
}

// x_perm[p] = x[sorted_token[p]]: one row per block-iteration, 16-byte vectors
__global__ void gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ sorted_token,
                                   uint4* __restrict__ xp, long long S, int T, int vec_per_row, uint32_t* err) {
    for (long long p = blockIdx.x; p < S; p += gridDim.x) {
        const int t = sorted_token[p];
        const bool ok = t >= 0 && t < T;
        if (!ok && threadIdx.x == 0) flag_error(err, ERR_INDEX_RANGE);
        const uint4* src = x + (size_t)(ok ? t : 0) * vec_per_row;
        uint4* dst = xp + (size_t)p * vec_per_row;
        for (int v = threadIdx.x; v < vec_per_row; v += blockDim.x) dst[v] = ok ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
    }
}

// x_perm[slot_of[t*k + j]] = x[t] for every pick j of token t: the same rows as
// gather_rows_kernel, written in token order, so each row of x is read from HBM once and
// stored k times (a gather re-reads each token's row k times from scattered places, mostly
// from HBM, since the sorted order visits a token once per expert it picked).  One block per
// token: the k destinations go to shared memory, then each thread moves 16-byte vectors.  A
// position outside [0, S) sets bit 4 and is skipped; a dropped slot (-1) is skipped.
__global__ void __launch_bounds__(128) scatter_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ slot_of,
                                                           uint4* __restrict__ xp, int T, int k, long long S,
                                                           int vec_per_row, uint32_t* err) {
    __shared__ int dst[32];
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();
        if ((int)threadIdx.x < k) {
            int p = slot_of[(size_t)t * k + threadIdx.x];
            if (p >= S) { flag_error(err, ERR_INDEX_RANGE); p = -1; }
            dst[threadIdx.x] = p;
        }
        __syncthreads();
        const uint4* src = x + (size_t)t * vec_per_row;
        for (int v = threadIdx.x; v < vec_per_row; v += blockDim.x) {
            const uint4 val = __ldg(src + v);
            for (int j = 0; j < k; ++j) {
                const int p = dst[j];
                if (p >= 0) xp[(size_t)p * vec_per_row + v] = val;
            }
        }
    }
}

// out[t] = base[t] + sum_j y[slot_of[t*k + j]]: the shared experts' fp32 output (optional)
// first, then the routed rows in ascending pick order, summed in fp32 and rounded once.  One
// block per token: its slot rows are read as whole contiguous rows, V elements (16 bytes)
// per thread step; with k <= KF all k row loads of a step are issued before they are summed.
template <typename T, int V, int KF>
__global__ void __launch_bounds__(128) combine_kernel(const T* __restrict__ y, const int32_t* __restrict__ slot_of,
                                                      const float* __restrict__ base, T* __restrict__ out, int Tn,
                                                      int d, int k, long long S, uint32_t* err) {
    struct alignas(sizeof(T) * V) Vec { T e[V]; };
    __shared__ int sl[32];
    const int nv = d / V;
    for (int t = blockIdx.x; t < Tn; t += gridDim.x) {
        __syncthreads();
        if ((int)threadIdx.x < k) {
            int p = slot_of[(size_t)t * k + threadIdx.x];
            if (p < 0 || p >= S) { flag_error(err, ERR_INDEX_RANGE); p = -1; }
            sl[threadIdx.x] = p;
        }
        __syncthreads();
        for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < nv; v += blockDim.x * gridDim.y) {
            float acc[V];
            if (base && V % 4 == 0) {            // 16-byte loads (d % V == 0, base 16-byte aligned)
                const float4* b4 = reinterpret_cast<const float4*>(base + (size_t)t * d + (size_t)v * V);
#pragma unroll
                for (int i = 0; i < V / 4; ++i) {
                    const float4 f = b4[i];
                    acc[4 * i] = f.x; acc[4 * i + 1] = f.y; acc[4 * i + 2] = f.z; acc[4 * i + 3] = f.w;
                }
            } else if (base) {
#pragma unroll
                for (int i = 0; i < V; ++i) acc[i] = base[(size_t)t * d + (size_t)v * V + i];
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i) acc[i] = 0.f;
            }
            if (KF > 0) {
                Vec raw[KF > 0 ? KF : 1];
#pragma unroll
                for (int j = 0; j < KF; ++j) {
                    if (j < k && sl[j] >= 0) raw[j] = reinterpret_cast<const Vec*>(y + (size_t)sl[j] * d)[v];
                    else
#pragma unroll
                        for (int i = 0; i < V; ++i) raw[j].e[i] = from_f32<T>(0.f);
                }
#pragma unroll
                for (int j = 0; j < KF; ++j)
#pragma unroll
                    for (int i = 0; i < V; ++i) acc[i] += to_f32(raw[j].e[i]);
            } else {
                for (int j = 0; j < k; ++j) {
                    if (sl[j] < 0) continue;
                    const Vec raw = reinterpret_cast<const Vec*>(y + (size_t)sl[j] * d)[v];
#pragma unroll
                    for (int i = 0; i < V; ++i) acc[i] += to_f32(raw.e[i]);
                }
            }
            Vec o;
#pragma unroll
            for (int i = 0; i < V; ++i) o.e[i] = from_f32<T>(acc[i]);
            reinterpret_cast<Vec*>(out + (size_t)t * d)[v] = o;
        }
    }
}

}  // namespace

cudaError_t launch_permute(const Dims& D, const int32_t* idx, const float* gate, int32_t* counts, int32_t* offsets,
                           int32_t* sorted_token, float* sorted_gate, int32_t* slot_of, int32_t* block_hist,
                           uint32_t* err, cudaStream_t stream) {
    const long long S = D.slots();
    if (permute_small(D)) {
        const size_t smem = sizeof(int) * (33 * (size_t)D.E + 32);
        permute_small_kernel<<<1, 1024, smem, stream>>>(idx, gate, S, D.k, D.E, counts, offsets, sorted_token,
                                                        sorted_gate, slot_of, err);
        return cudaGetLastError();
    }
    const int nblk = permute_blocks(D);
    const size_t smemE = sizeof(int) * D.E;
    if (nblk > 0) {
        permute_hist_kernel<<<nblk, 256, smemE, stream>>>(idx, S, D.E, block_hist, err);
    }
    permute_scan_kernel<<<1, SCAN_THREADS, smemE + 32 * sizeof(int), stream>>>(block_hist, nblk, D.E, counts, offsets);
    if (nblk > 0) {
        permute_scatter_kernel<<<nblk, 32, smemE, stream>>>(idx, gate, S, D.k, D.E, block_hist, sorted_token,
                                                            sorted_gate, slot_of);
    }
    return cudaGetLastError();
}

cudaError_t launch_plan(const Dims& D, const int32_t* offsets, int32_t* tile_start1, int32_t* tile_start2,
                        uint32_t* err, cudaStream_t stream) {
    const int G = D.E + D.Ks;
    const size_t smem = sizeof(int) * ((size_t)G + 1 + D.E + 1 + 32);
    plan_kernel<<<1, SCAN_THREADS, smem, stream>>>(offsets, D.slots(), D.T, D.d, D.E, D.I, D.Ks, D.Ks > 0 ? D.Is : 1,
                                                   gemm_tile_rows(D),
                                                   tile_start1, tile_start2, err);
    return cudaGetLastError();
}

cudaError_t launch_gather(const Dims& D, const void* x, const int32_t* sorted_token, void* x_perm, uint32_t* err,
                          cudaStream_t stream) {
    const long long S = D.slots();
    if (S == 0) return cudaSuccess;
    const int esz = D.bf16 ? 2 : 4;
    const int vec = D.d * esz / 16;
    const long long blocks = S < 148LL * 32 ? S : 148LL * 32;
    gather_rows_kernel<<<(int)blocks, 128, 0, stream>>>((const uint4*)x, sorted_token, (uint4*)x_perm, S, D.T, vec, err);
    return cudaGetLastError();
}

cudaError_t launch_scatter_rows(const Dims& D, const void* x, const int32_t* slot_of, void* x_perm, uint32_t* err,
                                cudaStream_t stream) {
    if (D.T == 0) return cudaSuccess;
    const int esz = D.bf16 ? 2 : 4;
    const int vec = D.d * esz / 16;
    const int blocks = D.T < 148 * 16 ? D.T : 148 * 16;
    scatter_rows_kernel<<<blocks, 128, 0, stream>>>((const uint4*)x, slot_of, (uint4*)x_perm, D.T, D.k, D.slots(), vec,
                                                    err);
    return cudaGetLastError();
}

// The grid is the number of blocks that fit on the GPU at once (one wave; each block loops over
// tokens), so no partial last wave leaves most SMs idle while a few finish their tokens.  With few
// tokens (decode) the grid's y dimension also splits each row's columns, so that every thread's
// loads are in flight at once instead of one column step after another.
template <typename K>
int resident_blocks(K kern, int threads) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    return per_sm * num_sms();
}

template <typename T, int V>
void combine_dispatch(const Dims& D, const void* y, const int32_t* slot_of, const float* base, void* out, uint32_t* err,
                      cudaStream_t stream) {
    const int nv = D.d / V;
    const int chunks = (nv + 127) / 128;
    if (D.k <= 8) {
        static const int cap = resident_blocks(combine_kernel<T, V, 8>, 128);
        const dim3 grid(D.T < cap ? D.T : cap, (long long)D.T * chunks <= 2LL * cap ? chunks : 1);
        combine_kernel<T, V, 8><<<grid, 128, 0, stream>>>((const T*)y, slot_of, base, (T*)out, D.T, D.d, D.k,
                                                          D.slots(), err);
    } else {
        static const int cap = resident_blocks(combine_kernel<T, V, 0>, 128);
        const dim3 grid(D.T < cap ? D.T : cap, (long long)D.T * chunks <= 2LL * cap ? chunks : 1);
        combine_kernel<T, V, 0><<<grid, 128, 0, stream>>>((const T*)y, slot_of, base, (T*)out, D.T, D.d, D.k,
                                                          D.slots(), err);
    }
}

cudaError_t launch_combine(const Dims& D, const void* y_sorted, const int32_t* slot_of, const float* base, void* out,
                           uint32_t* err, cudaStream_t stream) {
    if (D.T == 0) return cudaSuccess;
    if (D.bf16 && D.d % 8 == 0) combine_dispatch<__nv_bfloat16, 8>(D, y_sorted, slot_of, base, out, err, stream);
    else if (D.bf16) combine_dispatch<__nv_bfloat16, 1>(D, y_sorted, slot_of, base, out, err, stream);
    else if (D.d % 4 == 0) combine_dispatch<float, 4>(D, y_sorted, slot_of, base, out, err, stream);
    else combine_dispatch<float, 1>(D, y_sorted, slot_of, base, out, err, stream);
    return cudaGetLastError();
}

}  // namespace moe
