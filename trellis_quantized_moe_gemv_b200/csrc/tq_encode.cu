// T16 tail-biting Viterbi encoder (trellis_encode): finds, for every 16x16 tile of a
// target matrix, a K-bit-per-weight bit stream whose T16 codes are close to the
// targets in squared error.
//
// Method: "DeepSeek-V4.1-Flash-1017 · dsx T16", "How T16 works" -- the experts' streams
// are a bitshift trellis found by a Viterbi search (item 1's codebook, item 2's tile
// positions, item 4: a quantizer that minimises squared error).  The search rules the
// card leaves open are fixed as follows:
//   * objective per tile: sum_p (tau_p - 4 c_p)^2 over the 256 positions, tau_p =
//     rint(4 * target_p) clamped to [-1276, 1276] (quarter code units, exact integers,
//     < 2^32 per path), c_p = t(w_p) - 255 the centred code of window p;
//   * trellis: state = the 16-bit window; w_{p+1} = (w_p >> K) | (u << (16-K)); the
//     stream is tail-biting: w_0's low 16-K bits are w_255's high 16-K bits;
//   * pass 1 with free start and end; if its best path closes, done; otherwise two
//     closed passes with the closure bits b = w_255 >> K and b = w_0 & (2^(16-K) - 1)
//     of pass 1's path (window 0 restricted to low bits b, final window to high bits
//     b); the cheaper wins, the first on a tie.  Ties inside a pass go to the smaller
//     dropped bits and to the smaller final window.
//
// One CTA of 1024 threads per tile (persistent over tiles).  The predecessors of window
// s are the 2^K windows (m << K) | d with m = s & (2^(16-K) - 1), and they are
// consecutive, so a step is: for each group of 2^K consecutive windows, a thread forms
// their path costs from best[m] (shared memory, double-buffered) plus
// (tau_p - 4 c(s))^2 and reduces them into the next best[] and the backpointers (the
// winning d of every m, one byte, in the CTA's global workspace rows).  The traceback walks the
// backpointer rows from the chosen final window; the stream bits are assembled with warp
// ballots.  Integer arithmetic throughout, so the result is exactly the oracle's.
#include "tq_common.cuh"

namespace tq {

constexpr int kEncThreads = 1024;
constexpr int kEncPos = 256;             // positions per tile
constexpr int kEncPer = 65536 / kEncThreads;   // windows per thread
constexpr int kTauMax = 1276;
constexpr uint32_t kEncBig = 1u << 31;   // start cost of a window a closed pass excludes

template <int K>
struct EncShape {
    static constexpr int G = 1 << K;             // predecessors per group
    static constexpr int M = 1 << (16 - K);      // groups (low 16-K bits)
    static constexpr uint32_t kMask = M - 1;
    static constexpr int kGroups = kEncPer / G;  // groups per thread
};

template <int K>
struct EncSmem {
    uint32_t best[2][EncShape<K>::M];
    int tau[kEncPos];
    int w[3][kEncPos];                    // paths: pass 1, closed on b_end, closed on b_start
    unsigned long long red[kEncThreads / 32];
};

// Centred T16 code of window s, times 4, plus the 1020 offset folded into tau:
// (tau - 4 c)^2 = ((tau + 1020) - 4 t)^2 with t = lo + hi of (s * 0x3A2F) mod 2^16.
__device__ __forceinline__ uint32_t enc_dist(uint32_t s, int tq) {
    const uint32_t prod = (s * kT16Mult) & 0xFFFFu;
    const int t = (int)((prod & 0xFFu) + (prod >> 8));
    const int diff = tq - 4 * t;
    return (uint32_t)(diff * diff);
}

// One pass over the tile's positions.  b < 0: free start and end; else closed on b.
// Writes the backpointer rows bp[p][m] (p = 0..254) and returns the best allowed final
// window and its cost.  Thread t handles the groups (2^K consecutive windows with the
// same high bits) t, t + 1024, t + 2048, ...: a warp reads 32 consecutive groups'
// minima from best[] and writes 32 consecutive results, free of bank conflicts.
template <int K>
__device__ void enc_pass(EncSmem<K> &sm, int b, uint8_t *__restrict__ bp, uint32_t &out_cost, int &out_last) {
    using S = EncShape<K>;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned long long key = ~0ull;
    for (int p = 0; p < kEncPos; ++p) {
        const int tq = sm.tau[p] + 1020;
        const uint32_t *prev = sm.best[(p + 1) & 1];
        uint32_t *next = sm.best[p & 1];
        uint8_t *row = bp + (size_t)p * S::M;
#pragma unroll 1
        for (int j = 0; j < S::kGroups; ++j) {
            const uint32_t gi = (uint32_t)j * kEncThreads + tid;   // group: windows gi*G + d
            const uint32_t s = gi * S::G;
            const uint32_t m0 = s & S::kMask;
            uint32_t c[S::G];
#pragma unroll
            for (int d = 0; d < S::G; d += 4) {
                uint4 base4;
                if (p == 0) {   // start: free, or window 0's low bits equal to b
                    base4.x = (b < 0 || ((s + d + 0) & S::kMask) == (uint32_t)b) ? 0u : kEncBig;
                    base4.y = (b < 0 || ((s + d + 1) & S::kMask) == (uint32_t)b) ? 0u : kEncBig;
                    base4.z = (b < 0 || ((s + d + 2) & S::kMask) == (uint32_t)b) ? 0u : kEncBig;
                    base4.w = (b < 0 || ((s + d + 3) & S::kMask) == (uint32_t)b) ? 0u : kEncBig;
                } else {
                    base4 = *reinterpret_cast<const uint4 *>(prev + m0 + d);
                }
                c[d] = base4.x + enc_dist(s + d, tq);
                c[d + 1] = base4.y + enc_dist(s + d + 1, tq);
                c[d + 2] = base4.z + enc_dist(s + d + 2, tq);
                c[d + 3] = base4.w + enc_dist(s + d + 3, tq);
            }
            if (p < kEncPos - 1) {
                // pairwise minimum, the left (smaller d) kept on a tie
                uint32_t a[S::G];
#pragma unroll
                for (int d = 0; d < S::G; ++d) a[d] = d;
#pragma unroll
                for (int w = 1; w < S::G; w <<= 1)
#pragma unroll
                    for (int d = 0; d < S::G; d += 2 * w)
                        if (c[d + w] < c[d]) {
                            c[d] = c[d + w];
                            a[d] = a[d + w];
                        }
                next[gi] = c[0];
                row[gi] = (uint8_t)a[0];
            } else {
#pragma unroll
                for (int d = 0; d < S::G; ++d) {
                    if (b >= 0 && (int)((s + d) >> K) != b) continue;
                    const unsigned long long k = ((unsigned long long)c[d] << 16) | (s + d);
                    key = k < key ? k : key;
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
        key = other < key ? other : key;
    }
    if (lane == 0) sm.red[warp] = key;
    __syncthreads();
    if (tid == 0) {
        unsigned long long k = sm.red[0];
        for (int i = 1; i < kEncThreads / 32; ++i) k = sm.red[i] < k ? sm.red[i] : k;
        sm.red[0] = k;
    }
    __syncthreads();
    const unsigned long long k = sm.red[0];
    out_cost = (uint32_t)(k >> 16);
    out_last = (int)(k & 0xFFFFu);
    __syncthreads();
}

// Path windows w[0..255] from the final window, by the backpointer rows (thread 0).
// The rows were written by the CTA's threads in this launch; they are read after a
// barrier through a volatile pointer (never the read-only path).
template <int K>
__device__ void enc_traceback(const volatile uint8_t *bp, int last, int *w) {
    using S = EncShape<K>;
    if (threadIdx.x == 0) {
        int cur = last;
        w[kEncPos - 1] = cur;
        for (int p = kEncPos - 1; p > 0; --p) {
            const int m = cur & (int)S::kMask;
            cur = (m << K) | (int)bp[(size_t)(p - 1) * S::M + m];
            w[p - 1] = cur;
        }
    }
    __syncthreads();
}

template <int K>
__global__ void __launch_bounds__(kEncThreads, 1)
    trellis_encode_kernel(const float *__restrict__ target, int rows, int cols, uint32_t *__restrict__ bits,
                          uint32_t *__restrict__ tile_cost, uint8_t *__restrict__ ws) {
    using S = EncShape<K>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    EncSmem<K> &sm = *reinterpret_cast<EncSmem<K> *>(smem_raw);
    uint8_t *bp = ws + (size_t)blockIdx.x * (kEncPos - 1) * S::M;
    const int tid = threadIdx.x, lane = tid & 31;
    const int tcols = cols / 16, tiles = (rows / 16) * tcols;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int ti = tile / tcols, tj = tile - ti * tcols;
        if (tid < kEncPos) {   // position p = 16 * column + row inside the tile
            const float x = target[(size_t)(16 * ti + (tid & 15)) * cols + 16 * tj + (tid >> 4)];
            const int q = __float2int_rn(4.0f * x);
            sm.tau[tid] = max(-kTauMax, min(kTauMax, q));
        }
        __syncthreads();
        uint32_t cost;
        int last;
        enc_pass<K>(sm, -1, bp, cost, last);
        enc_traceback<K>(bp, last, sm.w[0]);
        const int b_end = sm.w[0][kEncPos - 1] >> K, b_start = sm.w[0][0] & (int)S::kMask;
        int pick = 0;
        if (b_end != b_start) {
            uint32_t ca, cb;
            int la, lb;
            enc_pass<K>(sm, b_end, bp, ca, la);
            enc_traceback<K>(bp, la, sm.w[1]);
            enc_pass<K>(sm, b_start, bp, cb, lb);
            enc_traceback<K>(bp, lb, sm.w[2]);
            pick = ca <= cb ? 1 : 2;
            cost = ca <= cb ? ca : cb;
        }
        // stream bit j = bit (j - pK) of w_p, p = j / K; one warp ballot per word
        const int *w = sm.w[pick];
        uint32_t *out = bits + (size_t)tile * (8 * K);
        if (tid < kEncPos * K) {
            const int p = tid / K;
            const bool bit = (w[p] >> (tid - p * K)) & 1;
            const unsigned word = __ballot_sync(0xffffffffu, bit);
            if (lane == 0) out[tid >> 5] = word;
        }
        if (tid == 0 && tile_cost) tile_cost[tile] = cost;
        __syncthreads();
    }
}

template <int K>
size_t enc_smem() {
    return sizeof(EncSmem<K>);
}

// CTAs resident at once (one per SM: the kernel takes 1024 threads and the K = 2 form
// 129 KB of shared memory) and the workspace they need: 255 backpointer rows each.
inline int enc_ctas(long long tiles) {
    return (int)max(1ll, min(tiles, (long long)num_sms()));
}

inline size_t enc_ws_bytes(int K, long long tiles) {
    return (size_t)enc_ctas(tiles) * (kEncPos - 1) * ((size_t)1 << (16 - K));
}

template <int K>
int run_encode(const float *target, int rows, int cols, uint32_t *bits, uint32_t *tile_cost, uint8_t *ws,
               cudaStream_t s) {
    static PerDeviceFlag configured;
    if (!configured.get()) {
        if (cudaFuncSetAttribute(trellis_encode_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)enc_smem<K>()) != cudaSuccess)
            return record_cuda_error("cudaFuncSetAttribute");
        configured.set();
    }
    const long long tiles = (long long)(rows / 16) * (cols / 16);
    LaunchScope ls(s, kStageEncode);
    trellis_encode_kernel<K><<<enc_ctas(tiles), kEncThreads, enc_smem<K>(), s>>>(target, rows, cols, bits,
                                                                                  tile_cost, ws);
    return launch_status();
}

}  // namespace tq

using namespace tq;

TQ_API size_t trellis_encode_workspace_size(int K, int rows, int cols) {
    if (K < 2 || K > 4 || rows < 0 || cols < 0 || rows % 16 || cols % 16) return 0;
    const long long tiles = (long long)(rows / 16) * (cols / 16);
    return tiles == 0 ? 0 : enc_ws_bytes(K, tiles);
}

TQ_API int trellis_encode(const float *target, int K, int rows, int cols, uint32_t *bits, uint32_t *tile_cost,
                          void *ws, size_t ws_bytes, tq_stream stream) {
    if (K < 2 || K > 4 || rows < 0 || cols < 0 || rows % 16 || cols % 16) return TQ_ERR_INVALID_ARG;
    const long long tiles = (long long)(rows / 16) * (cols / 16);
    if (tiles == 0) return TQ_OK;
    if (tiles > 0x7fffffffll) return TQ_ERR_UNSUPPORTED;
    if (!target || !bits || !ws) return TQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(target) & 3) || (reinterpret_cast<uintptr_t>(bits) & 3) ||
        (reinterpret_cast<uintptr_t>(tile_cost) & 3) || !aligned16(ws))
        return TQ_ERR_ALIGNMENT;
    if (ws_bytes < enc_ws_bytes(K, tiles)) return TQ_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t *w = reinterpret_cast<uint8_t *>(ws);
    if (K == 2) return run_encode<2>(target, rows, cols, bits, tile_cost, w, s);
    if (K == 3) return run_encode<3>(target, rows, cols, bits, tile_cost, w, s);
    return run_encode<4>(target, rows, cols, bits, tile_cost, w, s);
}
