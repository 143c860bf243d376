// Per-expert token lists, the grouped GEMMs' tile tables, the row gather and the combine.
//
// The grouping follows the "top-k indices first, then gather the tokens of each expert"
// step of the DeepSeek-V2 explainer (eliteato.com/news/32734, §3.1 and §3.3): the T*N_r
// slots (slot s = t*N_r + j) are grouped by expert in three passes — a per-block histogram,
// a scan over (expert, block), and a scatter that ranks equal experts inside a warp with
// __match_any_sync.  Inside an expert the slots keep ascending order, so the result does not
// depend on scheduling (no order-dependent atomics).
#include <atomic>

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

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
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

// The same token-order row move by the copy engine: one warp per block, lane 0 bringing each
// token's whole row into shared memory with one bulk copy (completion counted on an mbarrier)
// and storing it to the token's k slot positions with k bulk copies, two rows in flight per
// block (double buffer); lanes < k fetch the positions.  No data passes through registers.
// Waits on the load barriers are bounded (error bit 2, the remaining copies drained).
constexpr unsigned long long SCATTER_WAIT_NS = 1000000000ull;
__device__ __forceinline__ unsigned long long scatter_clock() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ bool scatter_wait(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = scatter_clock();
    for (uint32_t i = 0;; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
        if ((i & 63u) == 63u && (scatter_clock() - t0 > SCATTER_WAIT_NS || i >= (1u << 28))) return false;
    }
}
__global__ void __launch_bounds__(32) scatter_rows_bulk_kernel(const char* __restrict__ x,
                                                               const int32_t* __restrict__ slot_of,
                                                               char* __restrict__ xp, int T, int k, long long S,
                                                               uint32_t row_bytes, const float* __restrict__ sscale,
                                                               float* __restrict__ dscale, uint32_t* err) {
    extern __shared__ __align__(128) uint8_t rows[];           // two row buffers
    __shared__ __align__(8) uint64_t bars[2];
    const int lane = threadIdx.x;
    const uint32_t bar0 = (uint32_t)__cvta_generic_to_shared(&bars[0]);
    const uint32_t buf0 = (uint32_t)__cvta_generic_to_shared(rows);
    if (lane == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    const int n = (int)blockIdx.x < T ? (T - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    auto load = [&](int i) {                                    // lane 0: token i of this block into buffer i & 1
        const int t = (int)blockIdx.x + i * (int)gridDim.x;
        const uint32_t b = bar0 + 8u * (i & 1), dst = buf0 + row_bytes * (i & 1);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(row_bytes) : "memory");
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                     "l"(x + (size_t)t * row_bytes), "r"(row_bytes), "r"(b)
                     : "memory");
    };
    if (lane == 0 && n > 0) load(0);
    bool ok = true;
    int i = 0;
    for (; i < n; ++i) {
        const int t = (int)blockIdx.x + i * (int)gridDim.x;
        int pos = -1;
        if (lane < k) {
            pos = slot_of[(size_t)t * k + lane];
            if (pos >= S) { flag_error(err, ERR_INDEX_RANGE); pos = -1; }
            if (dscale && pos >= 0) dscale[pos] = sscale[t];   // row scale with the row (e4m3 codes)
        }
        if (lane == 0) {
            if (i + 1 < n) {
                // buffer (i + 1) & 1 was last read by token i - 1's stores: they must be done reading
                asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                load(i + 1);
            }
            ok = scatter_wait(bar0 + 8u * (i & 1), (uint32_t)((i >> 1) & 1));
            if (!ok) flag_error(err, ERR_PIPE_TIMEOUT);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        for (int j = 0; j < k; ++j) {
            const int pj = __shfl_sync(0xffffffffu, pos, j);
            if (lane == 0 && pj >= 0)
                asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(xp + (size_t)pj * row_bytes),
                             "r"(buf0 + row_bytes * (i & 1)), "r"(row_bytes)
                             : "memory");
        }
        if (lane == 0) asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    if (lane == 0) {
        if (!ok) {                                   // drain the loads still in flight (token i, and i + 1)
            scatter_wait(bar0 + 8u * (i & 1), (uint32_t)((i >> 1) & 1));
            if (i + 1 < n) scatter_wait(bar0 + 8u * ((i + 1) & 1), (uint32_t)(((i + 1) >> 1) & 1));
        }
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
    __syncwarp();
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

// The combine with its inputs staged by the copy engine: a persistent block walks (token, column
// chunk) items; thread 0 brings a chunk's k routed-row segments (bf16) and the shared output's
// segment (fp32) into one of two shared-memory stages with bulk copies counted on the stage's
// mbarrier, the whole block sums the next item while the following one is in flight, and each
// thread stores its 8 output columns.  The sum runs in the order of combine_kernel (base, then the
// picks in ascending j; with at most 8 picks absent ones add +0 as there), so the output is the
// same bit for bit.  Waits are bounded (error bit 2, the copies in flight drained).
constexpr int CB_COLS = 1024;                  // columns per chunk (8 per thread, 128 threads)
__global__ void __launch_bounds__(128) combine_bulk_kernel(const __nv_bfloat16* __restrict__ y,
                                                           const int32_t* __restrict__ slot_of,
                                                           const float* __restrict__ base,
                                                           __nv_bfloat16* __restrict__ out, int Tn, int d, int k,
                                                           long long S, uint32_t* err) {
    extern __shared__ __align__(128) uint8_t stage_mem[];
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ int pos_s[2][32];
    __shared__ int abort_s;
    const int tid = threadIdx.x;
    const int nch = (d + CB_COLS - 1) / CB_COLS;
    const uint32_t rows_bytes = (uint32_t)k * CB_COLS * 2;                 // routed segments of a stage
    const uint32_t stage_bytes = rows_bytes + (base ? CB_COLS * 4u : 0u);
    const uint32_t bar0 = (uint32_t)__cvta_generic_to_shared(&bars[0]);
    const uint32_t st0 = (uint32_t)__cvta_generic_to_shared(stage_mem);
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        abort_s = 0;
    }
    __syncthreads();
    // items of this block: token blockIdx.x + u * gridDim.x, chunk c, in (token, chunk) order
    const int ntok = (int)blockIdx.x < Tn ? (Tn - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int n = ntok * nch;
    auto issue = [&](int i) {                                  // thread 0: item i into stage i & 1
        const int t = (int)blockIdx.x + (i / nch) * (int)gridDim.x;
        const int c0 = (i % nch) * CB_COLS;
        const int cb = min(CB_COLS, d - c0);
        const int sidx = i & 1;
        const uint32_t b = bar0 + 8u * sidx, dst = st0 + stage_bytes * sidx;
        uint32_t bytes = 0;
        for (int j = 0; j < k; ++j) {
            int p = slot_of[(size_t)t * k + j];
            if (p >= S) { flag_error(err, ERR_INDEX_RANGE); p = -1; }
            else if (p < 0) { if (c0 == 0) flag_error(err, ERR_INDEX_RANGE); p = -1; }
            pos_s[sidx][j] = p;
            if (p >= 0) bytes += (uint32_t)cb * 2;
        }
        if (base) bytes += (uint32_t)cb * 4;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(bytes) : "memory");
        for (int j = 0; j < k; ++j) {
            const int p = pos_s[sidx][j];
            if (p >= 0)
                asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                                 dst + (uint32_t)j * CB_COLS * 2),
                             "l"(y + (size_t)p * d + c0), "r"((uint32_t)cb * 2), "r"(b)
                             : "memory");
        }
        if (base)
            asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                             dst + rows_bytes),
                         "l"(base + (size_t)t * d + c0), "r"((uint32_t)cb * 4), "r"(b)
                         : "memory");
    };
    if (tid == 0 && n > 0) issue(0);
    int i = 0;
    for (; i < n; ++i) {
        if (tid == 0 && i + 1 < n) issue(i + 1);               // its stage was released by the barrier below
        const int sidx = i & 1;
        if (!scatter_wait(bar0 + 8u * sidx, (uint32_t)((i >> 1) & 1))) {
            atomicExch(&abort_s, 1);
            flag_error(err, ERR_PIPE_TIMEOUT);
        }
        __syncthreads();
        if (abort_s) break;
        const int t = (int)blockIdx.x + (i / nch) * (int)gridDim.x;
        const int c0 = (i % nch) * CB_COLS;
        const int cb = min(CB_COLS, d - c0);
        const int col = tid * 8;
        if (col < cb) {
            const uint8_t* sb = stage_mem + (size_t)stage_bytes * sidx;
            float acc[8];
            if (base) {
                const float4* b4 = reinterpret_cast<const float4*>(sb + rows_bytes) + tid * 2;
                const float4 f0 = b4[0], f1 = b4[1];
                acc[0] = f0.x; acc[1] = f0.y; acc[2] = f0.z; acc[3] = f0.w;
                acc[4] = f1.x; acc[5] = f1.y; acc[6] = f1.z; acc[7] = f1.w;
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = 0.f;
            }
            const int jmax = k <= 8 ? 8 : k;
            for (int j = 0; j < jmax; ++j) {
                const bool live = j < k && pos_s[sidx][j] >= 0;
                if (!live && k > 8) continue;                  // as combine_kernel: zeros added only with <= 8 picks
                uint4 v = make_uint4(0, 0, 0, 0);
                if (live) v = *reinterpret_cast<const uint4*>(sb + (size_t)j * CB_COLS * 2 + (size_t)col * 2);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[2 * q] += __uint_as_float(w[q] << 16);
                    acc[2 * q + 1] += __uint_as_float(w[q] & 0xFFFF0000u);
                }
            }
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]); o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]); o.w = pack_bf16x2(acc[6], acc[7]);
            *reinterpret_cast<uint4*>(out + (size_t)t * d + c0 + col) = o;
        }
        __syncthreads();                                      // stage sidx free for item i + 2
    }
    if (tid == 0 && abort_s) {                                // drain what is still in flight
        scatter_wait(bar0 + 8u * (i & 1), (uint32_t)((i >> 1) & 1));
        if (i + 1 < n) scatter_wait(bar0 + 8u * ((i + 1) & 1), (uint32_t)(((i + 1) >> 1) & 1));
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

// Blocks of `kern` (threads, smem bytes) resident on the whole GPU, cached per shared-memory size
// (one entry per kernel instantiation: each call site passes its own cache).  The cached value only
// sizes persistent grids, so a stale or racing read changes the wave count, never the result.
template <typename K>
int resident_blocks_cached(K kern, int threads, int smem, std::atomic<unsigned long long>& cache) {
    const unsigned long long c = cache.load(std::memory_order_relaxed);
    if (c && (int)(c >> 32) == smem) return (int)(c & 0xFFFFFFFFu);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int n = per_sm * num_sms();
    cache.store(((unsigned long long)(unsigned)smem << 32) | (unsigned)n, std::memory_order_relaxed);
    return n;
}

cudaError_t launch_scatter_rows_bulk(const void* src, const float* sscale, const int32_t* slot_of, int T, int k,
                                     long long S, uint32_t row_bytes, void* dst, float* dscale, uint32_t* err,
                                     cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    if (row_bytes % 16 || row_bytes > 32768 || k > 32 || ((uintptr_t)src & 15u) || ((uintptr_t)dst & 15u) ||
        (dscale && !sscale))
        return cudaErrorNotSupported;
    static std::atomic<unsigned long long> cache{0};
    const int smem = 2 * (int)row_bytes;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(scatter_rows_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return cudaErrorInvalidValue;
    const int cap = resident_blocks_cached(scatter_rows_bulk_kernel, 32, smem, cache);
    scatter_rows_bulk_kernel<<<T < cap ? T : cap, 32, smem, stream>>>((const char*)src, slot_of, (char*)dst, T, k, S,
                                                                      row_bytes, sscale, dscale, err);
    return cudaGetLastError();
}

cudaError_t launch_scatter_rows(const Dims& D, const void* x, const int32_t* slot_of, void* x_perm, uint32_t* err,
                                cudaStream_t stream) {
    if (D.T == 0) return cudaSuccess;
    const int esz = D.bf16 ? 2 : 4;
    const uint32_t row_bytes = (uint32_t)D.d * esz;
    const cudaError_t e = launch_scatter_rows_bulk(x, nullptr, slot_of, D.T, D.k, D.slots(), row_bytes, x_perm, nullptr,
                                                   err, stream);
    if (e != cudaErrorNotSupported) return e;                  // else: rows not 16-byte aligned, register copy
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
    if (D.bf16 && D.d % 8 == 0 && D.k <= 32 && ((uintptr_t)y_sorted & 15u) == 0 && ((uintptr_t)out & 15u) == 0 &&
        ((uintptr_t)base & 15u) == 0) {
        static const int cap8 = resident_blocks(combine_kernel<__nv_bfloat16, 8, 8>, 128);
        const long long chunks = (D.d / 8 + 127) / 128;
        if (D.d >= 2048 && (long long)D.T * chunks > 2LL * cap8) {   // many tokens, long rows: bulk-staged inputs
            const int smem = 2 * (D.k * CB_COLS * 2 + (base ? CB_COLS * 4 : 0));
            if (cudaFuncSetAttribute(combine_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess)
                return cudaErrorInvalidValue;
            static std::atomic<unsigned long long> cache{0};
            const int cap = resident_blocks_cached(combine_bulk_kernel, 128, smem, cache);
            combine_bulk_kernel<<<D.T < cap ? D.T : cap, 128, smem, stream>>>(
                (const __nv_bfloat16*)y_sorted, slot_of, base, (__nv_bfloat16*)out, D.T, D.d, D.k, D.slots(), err);
            return cudaGetLastError();
        }
    }
    if (D.bf16 && D.d % 8 == 0) combine_dispatch<__nv_bfloat16, 8>(D, y_sorted, slot_of, base, out, err, stream);
    else if (D.bf16) combine_dispatch<__nv_bfloat16, 1>(D, y_sorted, slot_of, base, out, err, stream);
    else if (D.d % 4 == 0) combine_dispatch<float, 4>(D, y_sorted, slot_of, base, out, err, stream);
    else combine_dispatch<float, 1>(D, y_sorted, slot_of, base, out, err, stream);
    return cudaGetLastError();
}

}  // namespace moe
