// Routing: top-k + softmax, stable expert grouping, and the weighted combine.
//
// "top-8 softmax routing" of the routed experts; per-width groups with ascending
// global expert ids ("DeepSeek-V4.1-Flash-1017 TrellisMX K2 Mix", "What is stored").
#include "tq_combine.cuh"
#include "tq_common.cuh"

namespace tq {

constexpr int kTopkMaxPerLane = 32;   // E <= 32 * 32

// One warp per token.  Each lane owns logits e = lane + 32*j.  k rounds of a warp-wide
// arg-max (larger logit first, ties to the lower id) select the experts in order.
// The token's ids also go to ids_copy[lane] (lanes < k) when ids_copy is not null.
template <int PER_LANE>
__device__ __forceinline__ void topk_token(const float *__restrict__ logits, int token, int E, int k,
                                           int32_t *__restrict__ ids, float *__restrict__ w, int lane,
                                           int32_t *ids_copy) {
    const int warp = token;
    const float *row = logits + (size_t)warp * E;
    float v[PER_LANE];
#pragma unroll
    for (int j = 0; j < PER_LANE; ++j) {
        int e = lane + 32 * j;
        v[j] = e < E ? row[e] : -INFINITY;
    }
    uint32_t taken = 0;  // bit j: v[j] already selected (or absent)
#pragma unroll
    for (int j = 0; j < PER_LANE; ++j)
        if (lane + 32 * j >= E) taken |= 1u << j;
    float sel_v = 0.f, vmax = 0.f;
    int sel_e = 0;
    for (int r = 0; r < k; ++r) {
        // lane-local best (lowest id among equals: j ascending => id ascending)
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < PER_LANE; ++j) {
            bool free_slot = !((taken >> j) & 1u);
            if (free_slot && (v[j] > bv || be == 0x7fffffff)) {
                bv = v[j];
                be = lane + 32 * j;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        if (r == 0) vmax = bv;
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == r) {
            sel_v = bv;
            sel_e = be;
        }
    }
    // softmax over the k kept logits; lane r < k holds the r-th choice
    float ex = lane < k ? expf(sel_v - vmax) : 0.f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < k) {
        ids[(size_t)warp * k + lane] = sel_e;
        w[(size_t)warp * k + lane] = ex / sum;
        if (ids_copy) ids_copy[lane] = sel_e;
    }
}

template <int PER_LANE>
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ logits, int T,
                                                         int E, int k, int32_t *__restrict__ ids,
                                                         float *__restrict__ w) {
    chain_entry();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= T) return;
    topk_token<PER_LANE>(logits, warp, E, k, ids, w, lane, nullptr);
}

// Stable grouping of routes by expert in one CTA of 1024 threads.  Routes are taken
// in chunks of 1024 in index order; inside a chunk, a route's rank among equal
// experts is its rank inside its warp (match.any) plus the counts of the same expert
// in the chunk's earlier warps, plus the routes of that expert in earlier chunks.
constexpr int kPermThreads = 1024;
constexpr int kPermWarps = kPermThreads / 32;
constexpr int kPermMaxE = 1024;

__host__ __device__ inline size_t permute_smem_bytes(int E) {
    return sizeof(int32_t) * ((size_t)(3 + kPermWarps) * E);
}

// The grouping by one CTA of kPermThreads threads; smem holds permute_smem_bytes(E).
// topk_ids may point to global or shared memory.
__device__ __forceinline__ void permute_cta(const int32_t *topk_ids, int n_routes, int E,
                                            int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                                            int32_t *__restrict__ perm, int32_t *__restrict__ inv,
                                            int32_t *__restrict__ active_ids, int32_t *__restrict__ n_active,
                                            int32_t *smem) {
    int32_t *cursor = smem;                 // [E] histogram, then routes placed so far
    int32_t *base = cursor + E;             // [E] exclusive offsets
    int32_t *total = base + E;              // [E] routes of the current chunk
    int32_t *wcnt = total + E;              // [kPermWarps][E] per-warp counts of a chunk
    __shared__ int32_t warp_sum[kPermWarps], warp_sum_a[kPermWarps];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // per-warp count rows in use: warps past the routes of a chunk never write theirs
    const int wrows = min(kPermWarps, (n_routes + 31) / 32);
    for (int e = tid; e < E; e += kPermThreads) cursor[e] = 0;
    for (int x = tid; x < wrows * E; x += kPermThreads) wcnt[x] = 0;
    __syncthreads();
    bool bad = false;
    for (int i = tid; i < n_routes; i += kPermThreads) {
        int e = topk_ids[i];
        if (e >= 0 && e < E) atomicAdd(&cursor[e], 1);
        else bad = true;
    }
    if (bad) raise_flag(1);
    __syncthreads();

    // Exclusive scan of the histogram (one expert per thread) and of "expert active".
    const int c = tid < E ? cursor[tid] : 0;
    const int a = c > 0 ? 1 : 0;
    int incl = c, incl_a = a;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int t1 = __shfl_up_sync(0xffffffffu, incl, off);
        int t2 = __shfl_up_sync(0xffffffffu, incl_a, off);
        if (lane >= off) {
            incl += t1;
            incl_a += t2;
        }
    }
    if (lane == 31) {
        warp_sum[warp] = incl;
        warp_sum_a[warp] = incl_a;
    }
    __syncthreads();
    if (warp == 0) {
        int s = warp_sum[lane], sa = warp_sum_a[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int t1 = __shfl_up_sync(0xffffffffu, s, off);
            int t2 = __shfl_up_sync(0xffffffffu, sa, off);
            if (lane >= off) {
                s += t1;
                sa += t2;
            }
        }
        warp_sum[lane] = s;
        warp_sum_a[lane] = sa;
    }
    __syncthreads();
    const int prior = warp > 0 ? warp_sum[warp - 1] : 0;
    const int prior_a = warp > 0 ? warp_sum_a[warp - 1] : 0;
    if (tid < E) {
        const int ex = prior + incl - c;
        base[tid] = ex;
        offsets[tid] = ex;
        counts[tid] = c;
        if (c > 0) active_ids[prior_a + incl_a - 1] = tid;
        if (tid == E - 1) {
            offsets[E] = ex + c;
            *n_active = prior_a + incl_a;
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kPermThreads) cursor[e] = 0;
    __syncthreads();

    const unsigned lt_mask = (1u << lane) - 1u;
    for (int chunk = 0; chunk < n_routes; chunk += kPermThreads) {
        const int wmax = min(kPermWarps, (min(n_routes - chunk, kPermThreads) + 31) / 32);
        const int i = chunk + tid;
        const int e = i < n_routes ? topk_ids[i] : -1;
        const bool valid = e >= 0 && e < E;
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
        const int rank = __popc(peers & lt_mask);
        const bool leader = lane == 31 - __clz(peers);
        if (valid && leader) wcnt[warp * E + e] = __popc(peers);
        __syncthreads();
        for (int ee = tid; ee < E; ee += kPermThreads) {
            int run = 0;
            for (int w = 0; w < wmax; ++w) {
                const int v = wcnt[w * E + ee];
                wcnt[w * E + ee] = run;
                run += v;
            }
            total[ee] = run;
        }
        __syncthreads();
        if (valid) {
            const int dst = base[e] + cursor[e] + wcnt[warp * E + e] + rank;
            perm[dst] = i;
            inv[i] = dst;
        } else if (i < n_routes) {
            inv[i] = -1;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += kPermThreads) cursor[ee] += total[ee];
        for (int x = tid; x < wmax * E; x += kPermThreads) wcnt[x] = 0;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kPermThreads) route_permute_kernel(
    const int32_t *__restrict__ topk_ids, int n_routes, int E, int32_t *__restrict__ counts,
    int32_t *__restrict__ offsets, int32_t *__restrict__ perm, int32_t *__restrict__ inv,
    int32_t *__restrict__ active_ids, int32_t *__restrict__ n_active) {
    chain_entry();
    extern __shared__ int32_t smem[];
    permute_cta(topk_ids, n_routes, E, counts, offsets, perm, inv, active_ids, n_active, smem);
}

// Routing of a small batch in one launch: the 32 warps take the tokens' top-k in turn
// (writing ids and weights, and the ids into shared memory), then the CTA groups the
// routes from the shared copy -- the same results as route_topk then route_permute.
constexpr int kFusedRouteMax = 4096;    // routes (T*k) of one fused launch

template <int PER_LANE>
__global__ void __launch_bounds__(kPermThreads) route_topk_permute_kernel(
    const float *__restrict__ logits, int T, int E, int k, int32_t *__restrict__ ids, float *__restrict__ w,
    int32_t *__restrict__ counts, int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
    int32_t *__restrict__ inv, int32_t *__restrict__ active_ids, int32_t *__restrict__ n_active) {
    chain_entry();
    extern __shared__ int32_t smem[];
    int32_t *ids_s = smem + (permute_smem_bytes(E) / sizeof(int32_t));   // [T*k]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int t = warp; t < T; t += kPermWarps) topk_token<PER_LANE>(logits, t, E, k, ids, w, lane, ids_s + t * k);
    __syncthreads();
    permute_cta(ids_s, T * k, E, counts, offsets, perm, inv, active_ids, n_active, smem);
}

// ---------------------------------------------------------------- multi-CTA grouping
//
// The same stable grouping for large route counts in four launches, with no workspace:
// A: each block of kPermBlockRoutes routes counts its experts -> perm[b * E + e];
// B: one CTA turns those counts into each block's first position per expert
//    (offsets[e] + routes of e in earlier blocks) -> inv[b * E + e], and writes counts,
//    offsets and the active-expert list;
// C: each block reads its starting positions and places its routes exactly as the
//    single-CTA kernel does (chunks of 1024 in route order, match.any ranks), writing
//    perm only (inv still holds the starting positions other blocks read);
// D: inv[perm[j]] = j for the placed routes, -1 for routes with an invalid expert.
// perm and inv hold T*k >= blocks * E entries whenever T*k >= kPermMultiMin.
constexpr int kPermBlockRoutes = 4 * kPermThreads;
constexpr int kPermMultiMin = 16384;

__global__ void __launch_bounds__(kPermThreads) permute_hist_kernel(const int32_t *__restrict__ topk_ids,
                                                                    int n_routes, int E,
                                                                    int32_t *__restrict__ block_counts) {
    extern __shared__ int32_t hist[];
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += kPermThreads) hist[e] = 0;
    __syncthreads();
    const int r0 = blockIdx.x * kPermBlockRoutes, r1 = min(n_routes, r0 + kPermBlockRoutes);
    bool bad = false;
    for (int i = r0 + tid; i < r1; i += kPermThreads) {
        const int e = topk_ids[i];
        if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
        else bad = true;
    }
    if (bad) raise_flag(1);
    __syncthreads();
    for (int e = tid; e < E; e += kPermThreads) block_counts[(size_t)blockIdx.x * E + e] = hist[e];
}

__global__ void __launch_bounds__(kPermThreads) permute_scan_kernel(const int32_t *__restrict__ block_counts,
                                                                    int n_blocks, int E,
                                                                    int32_t *__restrict__ block_start,
                                                                    int32_t *__restrict__ counts,
                                                                    int32_t *__restrict__ offsets,
                                                                    int32_t *__restrict__ active_ids,
                                                                    int32_t *__restrict__ n_active) {
    __shared__ int32_t warp_sum[kPermWarps], warp_sum_a[kPermWarps];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int c = 0;
    if (tid < E)
        for (int b = 0; b < n_blocks; ++b) c += block_counts[(size_t)b * E + tid];
    const int a = c > 0 ? 1 : 0;
    int incl = c, incl_a = a;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int t1 = __shfl_up_sync(0xffffffffu, incl, off);
        const int t2 = __shfl_up_sync(0xffffffffu, incl_a, off);
        if (lane >= off) {
            incl += t1;
            incl_a += t2;
        }
    }
    if (lane == 31) {
        warp_sum[warp] = incl;
        warp_sum_a[warp] = incl_a;
    }
    __syncthreads();
    if (warp == 0) {
        int sm = warp_sum[lane], sa = warp_sum_a[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int t1 = __shfl_up_sync(0xffffffffu, sm, off);
            const int t2 = __shfl_up_sync(0xffffffffu, sa, off);
            if (lane >= off) {
                sm += t1;
                sa += t2;
            }
        }
        warp_sum[lane] = sm;
        warp_sum_a[lane] = sa;
    }
    __syncthreads();
    if (tid < E) {
        const int ex = (warp > 0 ? warp_sum[warp - 1] : 0) + incl - c;
        const int ex_a = (warp > 0 ? warp_sum_a[warp - 1] : 0) + incl_a - a;
        offsets[tid] = ex;
        counts[tid] = c;
        if (c > 0) active_ids[ex_a] = tid;
        if (tid == E - 1) {
            offsets[E] = ex + c;
            *n_active = ex_a + a;
        }
        // each block's first position for this expert, in block order
        int run = ex;
        for (int b = 0; b < n_blocks; ++b) {
            const int v = block_counts[(size_t)b * E + tid];
            block_start[(size_t)b * E + tid] = run;
            run += v;
        }
    }
}

__global__ void __launch_bounds__(kPermThreads) permute_scatter_kernel(const int32_t *__restrict__ topk_ids,
                                                                       int n_routes, int E,
                                                                       const int32_t *__restrict__ block_start,
                                                                       int32_t *__restrict__ perm) {
    extern __shared__ int32_t smem[];
    int32_t *cursor = smem;                 // [E] next position of each expert
    int32_t *total = cursor + E;            // [E] routes of the current chunk
    int32_t *wcnt = total + E;              // [kPermWarps][E] per-warp counts of a chunk
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < E; e += kPermThreads) cursor[e] = block_start[(size_t)blockIdx.x * E + e];
    for (int x = tid; x < kPermWarps * E; x += kPermThreads) wcnt[x] = 0;
    __syncthreads();
    const unsigned lt_mask = (1u << lane) - 1u;
    const int r0 = blockIdx.x * kPermBlockRoutes, r1 = min(n_routes, r0 + kPermBlockRoutes);
    for (int chunk = r0; chunk < r1; chunk += kPermThreads) {
        const int i = chunk + tid;
        const int e = i < r1 ? topk_ids[i] : -1;
        const bool valid = e >= 0 && e < E;
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
        const int rank = __popc(peers & lt_mask);
        const bool leader = lane == 31 - __clz(peers);
        if (valid && leader) wcnt[warp * E + e] = __popc(peers);
        __syncthreads();
        for (int ee = tid; ee < E; ee += kPermThreads) {
            int run = 0;
            for (int w = 0; w < kPermWarps; ++w) {
                const int v = wcnt[w * E + ee];
                wcnt[w * E + ee] = run;
                run += v;
            }
            total[ee] = run;
        }
        __syncthreads();
        if (valid) perm[cursor[e] + wcnt[warp * E + e] + rank] = i;
        __syncthreads();
        for (int ee = tid; ee < E; ee += kPermThreads) cursor[ee] += total[ee];
        for (int x = tid; x < kPermWarps * E; x += kPermThreads) wcnt[x] = 0;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(256) permute_inverse_kernel(const int32_t *__restrict__ topk_ids, int n_routes,
                                                              int E, const int32_t *__restrict__ offsets,
                                                              const int32_t *__restrict__ perm,
                                                              int32_t *__restrict__ inv) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= n_routes) return;
    if (j < offsets[E]) inv[perm[j]] = j;
    const int e = topk_ids[j];
    if (e < 0 || e >= E) inv[j] = -1;
}

static int route_permute_multi(const int32_t *topk_ids, int R, int E, int32_t *counts, int32_t *offsets,
                               int32_t *perm, int32_t *inv, int32_t *active_ids, int32_t *n_active,
                               cudaStream_t s) {
    static PerDeviceFlag configured;
    if (!configured.get()) {
        if (cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(sizeof(int32_t) * (2 + kPermWarps) * kPermMaxE)) != cudaSuccess)
            return TQ_ERR_CUDA;
        configured.set();
    }
    const int n_blocks = (R + kPermBlockRoutes - 1) / kPermBlockRoutes;
    {
        LaunchScope ls(s, kStagePermute);
        permute_hist_kernel<<<n_blocks, kPermThreads, sizeof(int32_t) * E, s>>>(topk_ids, R, E, perm);
    }
    int st = launch_status();
    if (st) return st;
    {
        LaunchScope ls(s, kStagePermute);
        permute_scan_kernel<<<1, kPermThreads, 0, s>>>(perm, n_blocks, E, inv, counts, offsets, active_ids, n_active);
    }
    if ((st = launch_status())) return st;
    {
        LaunchScope ls(s, kStagePermute);
        permute_scatter_kernel<<<n_blocks, kPermThreads, sizeof(int32_t) * (2 + kPermWarps) * E, s>>>(topk_ids, R, E,
                                                                                                  inv, perm);
    }
    if ((st = launch_status())) return st;
    LaunchScope ls(s, kStagePermute);
    permute_inverse_kernel<<<(R + 255) / 256, 256, 0, s>>>(topk_ids, R, E, offsets, perm, inv);
    return launch_status();
}

// out[t][d] = sum_s w[t][s] * y_perm[inv[t*k+s]][d], slot order, float4 per thread.
__global__ void __launch_bounds__(256) route_unpermute_kernel(const float *__restrict__ y_perm,
                                                              const int32_t *__restrict__ inv,
                                                              const float *__restrict__ w, int T,
                                                              int k, int D, int n_routes,
                                                              float *__restrict__ out) {
    chain_entry();
    const int d4 = D >> 2;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)T * d4) return;
    const int t = (int)(idx / d4);
    const int c = (int)(idx % d4);
    reinterpret_cast<float4 *>(out + (size_t)t * D)[c] = combine_slots(y_perm, inv, w, t, k, D, n_routes, 4 * c, true);
}

}  // namespace tq

using namespace tq;

TQ_API int route_topk(const float *logits, int T, int E, int k, int32_t *topk_ids, float *topk_w,
                      tq_stream stream) {
    if (T < 0 || k < 1 || k > 32 || E < k || E > 32 * kTopkMaxPerLane) return TQ_ERR_INVALID_ARG;
    if (T == 0) return TQ_OK;
    if (!logits || !topk_ids || !topk_w) return TQ_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const int threads = 256;
    const int blocks = (int)(((long long)T * 32 + threads - 1) / threads);
    const int per = (E + 31) / 32;
    LaunchScope ls(s, kStageTopk);
    if (per <= 4)
        launch_chained(route_topk_kernel<4>, blocks, threads, 0, s, logits, T, E, k, topk_ids, topk_w);
    else if (per <= 12)
        launch_chained(route_topk_kernel<12>, blocks, threads, 0, s, logits, T, E, k, topk_ids, topk_w);
    else
        launch_chained(route_topk_kernel<32>, blocks, threads, 0, s, logits, T, E, k, topk_ids, topk_w);
    return launch_status();
}

TQ_API int route_permute(const int32_t *topk_ids, int T, int k, int E, int32_t *counts,
                         int32_t *offsets, int32_t *perm, int32_t *inv, int32_t *active_ids,
                         int32_t *n_active, tq_stream stream) {
    if (T < 0 || k < 1 || E < 1 || E > kPermMaxE) return TQ_ERR_INVALID_ARG;
    if ((long long)T * k > (1ll << 30)) return TQ_ERR_UNSUPPORTED;
    if (!counts || !offsets || !active_ids || !n_active) return TQ_ERR_INVALID_ARG;
    if (T > 0 && (!topk_ids || !perm || !inv)) return TQ_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if ((long long)T * k >= kPermMultiMin)
        return route_permute_multi(topk_ids, T * k, E, counts, offsets, perm, inv, active_ids, n_active, s);
    const size_t smem = permute_smem_bytes(E);
    static PerDeviceFlag configured;
    if (!configured.get()) {
        if (cudaFuncSetAttribute(route_permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)permute_smem_bytes(kPermMaxE)) != cudaSuccess)
            return TQ_ERR_CUDA;
        configured.set();
    }
    LaunchScope ls(s, kStagePermute);
    launch_chained(route_permute_kernel, 1, kPermThreads, smem, s, topk_ids, T * k, E, counts, offsets, perm, inv,
                   active_ids, n_active);
    return launch_status();
}

TQ_API int route_topk_permute(const float *logits, int T, int E, int k, int32_t *topk_ids, float *topk_w,
                              int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv,
                              int32_t *active_ids, int32_t *n_active, tq_stream stream) {
    if (T < 0 || k < 1 || k > 32 || E < k || E > kPermMaxE) return TQ_ERR_INVALID_ARG;
    if ((long long)T * k > (1ll << 30)) return TQ_ERR_UNSUPPORTED;
    if (!counts || !offsets || !active_ids || !n_active) return TQ_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !topk_ids || !topk_w || !perm || !inv)) return TQ_ERR_INVALID_ARG;
    if ((long long)T * k > kFusedRouteMax || T == 0) {
        // large batches (and the empty one): the two launches
        int st = T > 0 ? route_topk(logits, T, E, k, topk_ids, topk_w, stream) : TQ_OK;
        if (st) return st;
        return route_permute(topk_ids, T, k, E, counts, offsets, perm, inv, active_ids, n_active, stream);
    }
    cudaStream_t s = (cudaStream_t)stream;
    const size_t smem = permute_smem_bytes(E) + sizeof(int32_t) * (size_t)T * k;
    static PerDeviceFlag configured;
    if (!configured.get()) {
        const int most = (int)(permute_smem_bytes(kPermMaxE) + sizeof(int32_t) * kFusedRouteMax);
        if (cudaFuncSetAttribute(route_topk_permute_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, most) !=
                cudaSuccess ||
            cudaFuncSetAttribute(route_topk_permute_kernel<12>, cudaFuncAttributeMaxDynamicSharedMemorySize, most) !=
                cudaSuccess ||
            cudaFuncSetAttribute(route_topk_permute_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, most) !=
                cudaSuccess)
            return TQ_ERR_CUDA;
        configured.set();
    }
    const int per = (E + 31) / 32;
    LaunchScope ls(s, kStageTopk);
    if (per <= 4)
        launch_chained(route_topk_permute_kernel<4>, 1, kPermThreads, smem, s, logits, T, E, k, topk_ids, topk_w,
                       counts, offsets, perm, inv, active_ids, n_active);
    else if (per <= 12)
        launch_chained(route_topk_permute_kernel<12>, 1, kPermThreads, smem, s, logits, T, E, k, topk_ids, topk_w,
                       counts, offsets, perm, inv, active_ids, n_active);
    else
        launch_chained(route_topk_permute_kernel<32>, 1, kPermThreads, smem, s, logits, T, E, k, topk_ids, topk_w,
                       counts, offsets, perm, inv, active_ids, n_active);
    return launch_status();
}

// Row gather for moving routed rows between layouts (expert-parallel dispatch and
// return): out[j] = src[index[j] / divisor], one 16-byte vector per thread.  An index
// outside [0, src_rows * divisor) raises device flag bit 0 and writes a zero row.
__global__ void __launch_bounds__(256) route_gather_rows_kernel(const uint4 *__restrict__ src, long long src_rows,
                                                                int row_vecs, const int32_t *__restrict__ index,
                                                                int divisor, long long rows,
                                                                uint4 *__restrict__ out) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= rows * row_vecs) return;
    const long long j = idx / row_vecs;
    const int c = (int)(idx % row_vecs);
    const int ix = index[j];
    const long long r = ix >= 0 ? ix / divisor : -1;
    if (r < 0 || r >= src_rows) {
        if (c == 0) raise_flag(1);
        out[idx] = make_uint4(0u, 0u, 0u, 0u);
        return;
    }
    out[idx] = src[r * row_vecs + c];
}

TQ_API int route_gather_rows(const void *src, int dtype, long long src_rows, int cols, const int32_t *index,
                             int divisor, long long rows, void *out, tq_stream stream) {
    if (dtype < TQ_DTYPE_F16 || dtype > TQ_DTYPE_F32 || src_rows < 0 || cols < 1 || divisor < 1 || rows < 0)
        return TQ_ERR_INVALID_ARG;
    const int esize = dtype == TQ_DTYPE_F32 ? 4 : 2;
    if (((long long)cols * esize) % 16) return TQ_ERR_INVALID_ARG;
    if (rows == 0) return TQ_OK;
    if (!src || !index || !out) return TQ_ERR_INVALID_ARG;
    if (!aligned16(src) || !aligned16(out)) return TQ_ERR_ALIGNMENT;
    const int row_vecs = (int)((long long)cols * esize / 16);
    const long long n = rows * row_vecs;
    if ((n + 255) / 256 > 0x7fffffffll) return TQ_ERR_UNSUPPORTED;
    cudaStream_t s = (cudaStream_t)stream;
    LaunchScope ls(s, kStageGather);
    route_gather_rows_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const uint4 *>(src), src_rows, row_vecs, index, divisor, rows, reinterpret_cast<uint4 *>(out));
    return launch_status();
}

TQ_API int route_unpermute(const float *y_perm, const int32_t *inv, const float *topk_w, int T,
                           int k, int D, float *out, tq_stream stream) {
    if (T < 0 || k < 1 || D < 4 || D % 4) return TQ_ERR_INVALID_ARG;
    if (T == 0) return TQ_OK;
    if (!y_perm || !inv || !topk_w || !out) return TQ_ERR_INVALID_ARG;
    if (!aligned16(y_perm) || !aligned16(out)) return TQ_ERR_ALIGNMENT;
    cudaStream_t s = (cudaStream_t)stream;
    const long long n = (long long)T * (D / 4);
    const int threads = 256;
    LaunchScope ls(s, kStageUnpermute);
    launch_chained(route_unpermute_kernel, (unsigned)((n + threads - 1) / threads), threads, 0, s, y_perm, inv,
                   topk_w, T, k, D, T * k, out);
    return launch_status();
}
