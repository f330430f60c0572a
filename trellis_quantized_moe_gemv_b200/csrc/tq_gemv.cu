// Decode-fused GEMV for T16 trellis-coded matrices: single projection (trellis_gemv)
// and the routed experts of a MoE layer for decode-sized batches (moe_trellis_gemv).
//
// Method: "DeepSeek-V4.1-Flash-1017 · dsx T16", "How T16 works" -- item 1 (T16: the
// 16-bit window times 0x3A2F mod 2^16, plus the product's two bytes), item 2
// (column-major 16x16 tiles), item 4 (per-output scales); gate/up/SiLU/down of the
// routed experts with fused gate/up post-processing ("October 25 runtime checkpoint").
//
// Decode in registers, contraction on the tensor cores (mma.sync, fp16 x fp16 -> fp32):
//   * A warp walks 8 strips (16 output rows each) at once: lane group g = lane/4 owns
//     strip g, so every lane decodes the same tile-relative bit offsets (compile-time
//     shifts) of its own tile; lane t = lane%4 owns columns 4t..4t+3 of each tile.
//   * Window -> product: R = bottom16(window) * 0x3A2F0000 + 0x6464 is one IMAD and
//     leaves [0x64, 0x64, lo, hi] (bytes 0..3) with lo/hi the two bytes of
//     (window*0x3A2F) mod 2^16.  One PRMT per weight interleaves lo (or hi) of two
//     weights with the 0x64 bytes: fp16 values 1024+lo, 1024+hi (exact).
//   * Two MMAs per tile (the lo plane and the hi plane) accumulate
//     sum_j (2048 + t_j) x_j in fp32; a third MMA with A = 1.0 accumulates sum_j x_j,
//     and the epilogue forms s * 2^-12 * (D - 2303 * sum_j x_j) = s * 2^-12 * sum_j c_j x_j.
//   * The 4 lanes of a strip split the tile's 8K words; the word after a lane's
//     quarter (tail-biting for the last quarter) comes from its neighbour by shuffle.
#include "tq_common.cuh"

namespace tq {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr uint32_t kSelLo = 0x4602u;   // [A.b2, A.b0, B.b2, B.b0] -> (1024+lo_A, 1024+lo_B)
constexpr uint32_t kSelHi = 0x5713u;   // [A.b3, A.b1, B.b3, B.b1] -> (1024+hi_A, 1024+hi_B)
constexpr uint32_t kOneH2 = 0x3C003C00u;
constexpr float kOffset = 2.0f * 1024.0f + 255.0f;   // (1024+lo)+(1024+hi) = c + 2303

// Packed T16 product of the window at compile-time bit offset O of the lane's span.
template <int O, int NS>
__device__ __forceinline__ uint32_t t16_pack(const uint32_t (&v)[NS]) {
    constexpr int wi = O >> 5, sh = O & 31;
    uint32_t bottom;
    if constexpr (sh == 0) bottom = v[wi];
    else bottom = funnel_r(v[wi], v[wi + 1], sh);
    return bottom * (kT16Mult << 16) + 0x6464u;
}

template <int NG>
struct Acc {
    float d[8][NG][4];   // [row pair][token group][fragment]
    float s[NG][4];      // sum of x per token (ones MMA)
};

// One column tile of the lane's strip: decode 64 windows (rows 0..15 x the lane's 4
// columns) and issue the MMAs for every token group.
template <int K, int NG, int P>
__device__ __forceinline__ void tile_pairs(const uint32_t (&v)[2 * K + 1], const uint2 (&xb)[NG],
                                           Acc<NG> &acc) {
    if constexpr (P < 8) {
        constexpr int r0 = P, r1 = P + 8;
        const uint32_t R00 = t16_pack<0 * 16 * K + K * r0>(v), R01 = t16_pack<1 * 16 * K + K * r0>(v);
        const uint32_t R02 = t16_pack<2 * 16 * K + K * r0>(v), R03 = t16_pack<3 * 16 * K + K * r0>(v);
        const uint32_t R10 = t16_pack<0 * 16 * K + K * r1>(v), R11 = t16_pack<1 * 16 * K + K * r1>(v);
        const uint32_t R12 = t16_pack<2 * 16 * K + K * r1>(v), R13 = t16_pack<3 * 16 * K + K * r1>(v);
        const uint32_t l0 = prmt(R00, R01, kSelLo), l1 = prmt(R10, R11, kSelLo);
        const uint32_t l2 = prmt(R02, R03, kSelLo), l3 = prmt(R12, R13, kSelLo);
        const uint32_t h0 = prmt(R00, R01, kSelHi), h1 = prmt(R10, R11, kSelHi);
        const uint32_t h2 = prmt(R02, R03, kSelHi), h3 = prmt(R12, R13, kSelHi);
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            mma_f16_16816(acc.d[P][g], l0, l1, l2, l3, xb[g].x, xb[g].y);
            mma_f16_16816(acc.d[P][g], h0, h1, h2, h3, xb[g].x, xb[g].y);
        }
        tile_pairs<K, NG, P + 1>(v, xb, acc);
    }
}

template <int K>
__device__ __forceinline__ void load_quarter(const uint32_t *p, uint32_t (&w)[2 * K]) {
    if constexpr (K == 2) {
        uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    } else if constexpr (K == 3) {
        uint2 a = __ldg(reinterpret_cast<const uint2 *>(p));
        uint2 b = __ldg(reinterpret_cast<const uint2 *>(p + 2));
        uint2 c = __ldg(reinterpret_cast<const uint2 *>(p + 4));
        w[0] = a.x; w[1] = a.y; w[2] = b.x; w[3] = b.y; w[4] = c.x; w[5] = c.y;
    } else {
        uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
        uint4 b = __ldg(reinterpret_cast<const uint4 *>(p + 4));
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
}

// Accumulate column tiles [jb, je) of the lane's strip (tile 0 of the strip at
// `strip0`, tiles 8K words apart) against the lane's token rows xr[g] (fp16, may be
// null: contributes zero).  Loads run PF tiles ahead.
template <int K, int NG>
__device__ __forceinline__ void accumulate(const uint32_t *__restrict__ strip0, int jb, int je,
                                           const __half *const (&xr)[NG], Acc<NG> &acc) {
    constexpr int PF = 2;
    constexpr int WPT = 8 * K;
    const int lane = threadIdx.x & 31, t4 = lane & 3;
    const int src = (lane & ~3) | ((lane + 1) & 3);
    const uint32_t *q0 = strip0 + 2 * K * t4;
    uint32_t buf[PF][2 * K];
    uint2 xb[PF][NG];
#pragma unroll
    for (int s = 0; s < PF; ++s) {
        if (jb + s < je) {
            load_quarter<K>(q0 + (size_t)(jb + s) * WPT, buf[s]);
#pragma unroll
            for (int g = 0; g < NG; ++g)
                xb[s][g] = xr[g] ? __ldg(reinterpret_cast<const uint2 *>(xr[g] + 16 * (jb + s) + 4 * t4))
                                 : make_uint2(0u, 0u);
        }
    }
    for (int j = jb; j < je; j += PF) {
#pragma unroll
        for (int s = 0; s < PF; ++s) {
            if (j + s < je) {
                uint32_t v[2 * K + 1];
#pragma unroll
                for (int i = 0; i < 2 * K; ++i) v[i] = buf[s][i];
                v[2 * K] = __shfl_sync(0xffffffffu, buf[s][0], src);
                uint2 x[NG];
#pragma unroll
                for (int g = 0; g < NG; ++g) x[g] = xb[s][g];
                const int jn = j + s + PF;
                if (jn < je) {
                    load_quarter<K>(q0 + (size_t)jn * WPT, buf[s]);
#pragma unroll
                    for (int g = 0; g < NG; ++g)
                        xb[s][g] = xr[g] ? __ldg(reinterpret_cast<const uint2 *>(xr[g] + 16 * jn + 4 * t4))
                                         : make_uint2(0u, 0u);
                }
                tile_pairs<K, NG, 0>(v, x, acc);
#pragma unroll
                for (int g = 0; g < NG; ++g)
                    mma_f16_16816(acc.s[g], kOneH2, kOneH2, kOneH2, kOneH2, x[g].x, x[g].y);
            }
        }
    }
}

template <int NG>
__device__ __forceinline__ void zero(Acc<NG> &acc) {
#pragma unroll
    for (int p = 0; p < 8; ++p)
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc.d[p][g][i] = 0.f;
#pragma unroll
    for (int g = 0; g < NG; ++g)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc.s[g][i] = 0.f;
}

// Shared-memory reduction buffers of one CTA.
template <int NG>
struct RedSmem {
    float d[kGemvWarps][NG][8][16][8];   // [warp][group][strip][row][token]
    float s[kGemvWarps][NG][8];          // [warp][group][token]
};

// Store the warp's partials: fragment (row g -> strip g row r0, row g+8 -> row r1,
// tokens 2t, 2t+1).
template <int NG>
__device__ __forceinline__ void store_partials(const Acc<NG> &acc, RedSmem<NG> &red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            red.d[warp][g][gq][p][2 * t4] = acc.d[p][g][0];
            red.d[warp][g][gq][p][2 * t4 + 1] = acc.d[p][g][1];
            red.d[warp][g][gq][p + 8][2 * t4] = acc.d[p][g][2];
            red.d[warp][g][gq][p + 8][2 * t4 + 1] = acc.d[p][g][3];
        }
        if (gq == 0) {
            red.s[warp][g][2 * t4] = acc.s[g][0];
            red.s[warp][g][2 * t4 + 1] = acc.s[g][1];
        }
    }
}

// Sum over warps in fixed order: raw accumulation of (strip, row, token, group).
template <int NG>
__device__ __forceinline__ float red_d(const RedSmem<NG> &red, int g, int strip, int row, int tok) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) v += red.d[w][g][strip][row][tok];
    return v;
}
template <int NG>
__device__ __forceinline__ float red_s(const RedSmem<NG> &red, int g, int tok) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) v += red.s[w][g][tok];
    return v;
}

__device__ __forceinline__ float finish(float d, float sx, float scale) {
    return scale * kKappa * (d - kOffset * sx);
}

__device__ __forceinline__ void split_range(int n, int part, int parts, int &b, int &e) {
    const int per = (n + parts - 1) / parts;
    b = min(n, part * per);
    e = min(n, b + per);
}

// --------------------------------------------------------------------------- single GEMV

// CTA = one group of 8 strips (128 rows) x a batch pass of 8*NG tokens; the 8 warps
// split the column tiles.
template <int K, int NG>
__global__ void __launch_bounds__(kGemvThreads, 2)
    trellis_gemv_kernel(const uint32_t *__restrict__ bits, const __half *__restrict__ scales, int rows,
                        int cols, const __half *__restrict__ x, int batch, float *__restrict__ y) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RedSmem<NG> &red = *reinterpret_cast<RedSmem<NG> *>(smem_raw);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gq = lane >> 2;
    const int n_strips = rows / 16, tiles = cols / 16;
    const int strip = blockIdx.x * 8 + gq;
    const int tok0 = blockIdx.y * 8 * NG;
    const uint32_t *strip0 =
        bits + (size_t)min(strip, n_strips - 1) * tiles * (8 * K);  // clamp: rows beyond are dropped
    const __half *xr[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        const int b = tok0 + 8 * g + gq;
        xr[g] = b < batch ? x + (size_t)b * cols : nullptr;
    }
    Acc<NG> acc;
    zero(acc);
    int jb, je;
    split_range(tiles, warp, kGemvWarps, jb, je);
    accumulate<K, NG>(strip0, jb, je, xr, acc);
    store_partials(acc, red);
    __syncthreads();
    for (int i = threadIdx.x; i < NG * 8 * 16 * 8; i += kGemvThreads) {
        const int tok = i & 7, row = (i >> 3) & 15, st = (i >> 7) & 7, g = i >> 10;
        const int b = tok0 + 8 * g + tok, r = (blockIdx.x * 8 + st) * 16 + row;
        if (b < batch && r < rows)
            y[(size_t)b * rows + r] =
                finish(red_d(red, g, st, row, tok), red_s(red, g, tok), __half2float(scales[r]));
    }
}

// --------------------------------------------------------------------------- MoE GEMV

struct ExpertRef {
    int K;
    const uint32_t *gate, *up, *down;
    const __half *s_gate, *s_up, *s_down;
};

__device__ __forceinline__ bool expert_ref(const tq_moe_layer &L, int e, ExpertRef &r) {
    if (e < 0 || e >= L.E) return false;
    const int slot = L.expert_slot[e];
    if (slot < 0) return false;
    const int gi = slot >> 16, idx = slot & 0xFFFF;
    if (gi >= L.n_groups) return false;
    const tq_width_group &G = L.groups[gi];
    if (idx >= G.n_experts) return false;
    const size_t words_proj = (size_t)(L.D / 16) * (L.F / 16) * 8 * G.K;
    r.K = G.K;
    r.gate = G.gate + (size_t)idx * words_proj;
    r.up = G.up + (size_t)idx * words_proj;
    r.down = G.down + (size_t)idx * words_proj;
    r.s_gate = reinterpret_cast<const __half *>(G.s_gate) + (size_t)idx * L.F;
    r.s_up = reinterpret_cast<const __half *>(G.s_up) + (size_t)idx * L.F;
    r.s_down = reinterpret_cast<const __half *>(G.s_down) + (size_t)idx * L.D;
    return true;
}

template <int NG>
__device__ __forceinline__ void accumulate_any_k(int K, const uint32_t *strip0, int jb, int je,
                                                 const __half *const (&xr)[NG], Acc<NG> &acc) {
    if (K == 2) accumulate<2, NG>(strip0, jb, je, xr, acc);
    else if (K == 3) accumulate<3, NG>(strip0, jb, je, xr, acc);
    else accumulate<4, NG>(strip0, jb, je, xr, acc);
}

// Gate/up + SiLU: item = (active expert, 64 intermediate rows).  Lane groups 0..3 walk
// gate strips, 4..7 the up strips of the same rows.  h[route][f] = silu(g) * u (fp32).
template <int NG>
__global__ void __launch_bounds__(kGemvThreads, 2)
    moe_gateup_kernel(const tq_moe_layer L, const __half *__restrict__ x_rot,
                      const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm,
                      const int32_t *__restrict__ active_ids, const int32_t *__restrict__ n_active_p,
                      int k, int n_routes, float *__restrict__ h) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RedSmem<NG> &red = *reinterpret_cast<RedSmem<NG> *>(smem_raw);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gq = lane >> 2;
    const int D = L.D, F = L.F, tiles = D / 16;
    const int items_per_expert = F / 64;
    const int n_items = *n_active_p * items_per_expert;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int a = item / items_per_expert, fi = item % items_per_expert;
        const int e = active_ids[a];
        ExpertRef ex;
        if (!expert_ref(L, e, ex)) {
            if (threadIdx.x == 0) raise_flag(1);
            continue;
        }
        const int r0 = offsets[e], ne = offsets[e + 1] - r0;
        const int f_strip = fi * 4 + (gq & 3);
        const uint32_t *proj = gq < 4 ? ex.gate : ex.up;
        const uint32_t *strip0 = proj + (size_t)f_strip * tiles * (8 * ex.K);
        for (int tb = 0; tb < ne; tb += 8 * NG) {
            const __half *xr[NG];
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const int tt = tb + 8 * g + gq;
                const int ri = r0 + tt;
                const int pr = tt < ne ? perm[ri] : -1;
                xr[g] = (pr >= 0 && pr < n_routes) ? x_rot + (size_t)(pr / k) * D : nullptr;
            }
            Acc<NG> acc;
            zero(acc);
            int jb, je;
            split_range(tiles, warp, kGemvWarps, jb, je);
            accumulate_any_k<NG>(ex.K, strip0, jb, je, xr, acc);
            __syncthreads();   // previous pass / item finished reading red
            store_partials(acc, red);
            __syncthreads();
            for (int i = threadIdx.x; i < NG * 4 * 16 * 8; i += kGemvThreads) {
                const int tok = i & 7, row = (i >> 3) & 15, st = (i >> 7) & 3, g = i >> 9;
                const int tt = tb + 8 * g + tok;
                if (tt >= ne) continue;
                const int f = (fi * 4 + st) * 16 + row;
                const float sx = red_s(red, g, tok);
                const float gv = finish(red_d(red, g, st, row, tok), sx, __half2float(ex.s_gate[f]));
                const float uv = finish(red_d(red, g, st + 4, row, tok), sx, __half2float(ex.s_up[f]));
                h[(size_t)(r0 + tt) * F + f] = silu_f32(gv) * uv;
            }
        }
    }
}

// Down projection: item = (active expert, 128 output rows).  y[route][d] = W_down h'.
template <int NG>
__global__ void __launch_bounds__(kGemvThreads, 2)
    moe_down_kernel(const tq_moe_layer L, const __half *__restrict__ h_rot,
                    const int32_t *__restrict__ offsets, const int32_t *__restrict__ active_ids,
                    const int32_t *__restrict__ n_active_p, float *__restrict__ y) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RedSmem<NG> &red = *reinterpret_cast<RedSmem<NG> *>(smem_raw);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gq = lane >> 2;
    const int D = L.D, F = L.F, tiles = F / 16;
    const int items_per_expert = D / 128;
    const int n_items = *n_active_p * items_per_expert;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int a = item / items_per_expert, di = item % items_per_expert;
        const int e = active_ids[a];
        ExpertRef ex;
        if (!expert_ref(L, e, ex)) {
            if (threadIdx.x == 0) raise_flag(1);
            continue;
        }
        const int r0 = offsets[e], ne = offsets[e + 1] - r0;
        const uint32_t *strip0 = ex.down + (size_t)(di * 8 + gq) * tiles * (8 * ex.K);
        for (int tb = 0; tb < ne; tb += 8 * NG) {
            const __half *xr[NG];
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const int tt = tb + 8 * g + gq;
                xr[g] = tt < ne ? h_rot + (size_t)(r0 + tt) * F : nullptr;
            }
            Acc<NG> acc;
            zero(acc);
            int jb, je;
            split_range(tiles, warp, kGemvWarps, jb, je);
            accumulate_any_k<NG>(ex.K, strip0, jb, je, xr, acc);
            __syncthreads();
            store_partials(acc, red);
            __syncthreads();
            for (int i = threadIdx.x; i < NG * 8 * 16 * 8; i += kGemvThreads) {
                const int tok = i & 7, row = (i >> 3) & 15, st = (i >> 7) & 7, g = i >> 10;
                const int tt = tb + 8 * g + tok;
                if (tt >= ne) continue;
                const int d = (di * 8 + st) * 16 + row;
                y[(size_t)(r0 + tt) * D + d] =
                    finish(red_d(red, g, st, row, tok), red_s(red, g, tok), __half2float(ex.s_down[d]));
            }
        }
    }
}

template <typename Kern>
inline int set_smem(Kern kern, size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) ==
                   cudaSuccess
               ? TQ_OK
               : TQ_ERR_CUDA;
}

inline size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

int validate_layer(const tq_moe_layer *L) {
    if (!L) return TQ_ERR_INVALID_ARG;
    if (L->E < 1 || L->E > 1024 || L->D < 128 || L->F < 128 || L->D % 128 || L->F % 128)
        return TQ_ERR_INVALID_ARG;
    if (L->n_groups < 1 || L->n_groups > 3 || !L->expert_slot) return TQ_ERR_INVALID_ARG;
    for (int g = 0; g < L->n_groups; ++g) {
        const tq_width_group &G = L->groups[g];
        if (G.K < 2 || G.K > 4 || G.n_experts < 0 || G.n_experts > 0xFFFF) return TQ_ERR_INVALID_ARG;
        if (G.n_experts == 0) continue;
        if (!G.gate || !G.up || !G.down || !G.s_gate || !G.s_up || !G.s_down) return TQ_ERR_INVALID_ARG;
        if (!aligned16(G.gate) || !aligned16(G.up) || !aligned16(G.down)) return TQ_ERR_ALIGNMENT;
    }
    return TQ_OK;
}

size_t workspace_bytes(const tq_moe_layer *L, int T, int k) {
    const size_t routes = (size_t)T * k;
    return align256(routes * L->F * sizeof(float)) + align256(routes * L->F * sizeof(__half));
}

int launch_hadamard128(const void *x, int x_dtype, long long rows, long long cols, __half *out,
                       cudaStream_t s, int stage);

template <int NG>
int run_moe_gemv(const tq_moe_layer *L, const __half *x_rot, const int32_t *offsets, const int32_t *perm,
                 const int32_t *active_ids, const int32_t *n_active, int T, int k, float *y_perm,
                 void *ws, cudaStream_t s) {
    const size_t smem = sizeof(RedSmem<NG>);
    static bool configured = false;
    if (!configured) {
        if (set_smem(moe_gateup_kernel<NG>, smem) || set_smem(moe_down_kernel<NG>, smem)) return TQ_ERR_CUDA;
        configured = true;
    }
    const int routes = T * k;
    float *h = reinterpret_cast<float *>(ws);
    __half *h_rot = reinterpret_cast<__half *>(reinterpret_cast<char *>(ws) +
                                               align256((size_t)routes * L->F * sizeof(float)));
    const int max_active = min(L->E, routes);
    const int grid_cap = 2 * num_sms();
    const int gu_items = max_active * (L->F / 64);
    const int dn_items = max_active * (L->D / 128);
    {
    LaunchScope ls(s, kStageGemvGateUp);
    moe_gateup_kernel<NG><<<min(gu_items, grid_cap), kGemvThreads, smem, s>>>(
        *L, x_rot, offsets, perm, active_ids, n_active, k, routes, h);
    }
    int st = launch_status();
    if (st) return st;
    st = launch_hadamard128(h, TQ_DTYPE_F32, routes, L->F, h_rot, s, kStageRotateH);
    if (st) return st;
    LaunchScope ls(s, kStageGemvDown);
    moe_down_kernel<NG><<<min(dn_items, grid_cap), kGemvThreads, smem, s>>>(*L, h_rot, offsets,
                                                                             active_ids, n_active, y_perm);
    return launch_status();
}

template <int K, int NG>
int run_gemv(const uint32_t *bits, const __half *scales, int rows, int cols, const __half *x, int batch,
             float *y, cudaStream_t s) {
    const size_t smem = sizeof(RedSmem<NG>);
    static bool configured = false;
    if (!configured) {
        if (set_smem(trellis_gemv_kernel<K, NG>, smem)) return TQ_ERR_CUDA;
        configured = true;
    }
    dim3 grid((rows / 16 + 7) / 8, (batch + 8 * NG - 1) / (8 * NG));
    LaunchScope ls(s, kStageGemv);
    trellis_gemv_kernel<K, NG><<<grid, kGemvThreads, smem, s>>>(bits, scales, rows, cols, x, batch, y);
    return launch_status();
}

}  // namespace tq

using namespace tq;

TQ_API int trellis_gemv(const uint32_t *bits, const uint16_t *scales, int K, int rows, int cols,
                        const uint16_t *x_rot, int batch, float *y, tq_stream stream) {
    if (K < 2 || K > 4 || rows < 0 || cols < 0 || rows % 16 || cols % 128 || batch < 0 || batch > 256)
        return TQ_ERR_INVALID_ARG;
    if (rows == 0 || batch == 0) return TQ_OK;
    if (cols == 0) return TQ_ERR_INVALID_ARG;
    if (!bits || !scales || !x_rot || !y) return TQ_ERR_INVALID_ARG;
    if (!aligned16(bits) || !aligned16(x_rot)) return TQ_ERR_ALIGNMENT;
    cudaStream_t s = (cudaStream_t)stream;
    const __half *sc = reinterpret_cast<const __half *>(scales);
    const __half *x = reinterpret_cast<const __half *>(x_rot);
    if (batch <= 8) {
        switch (K) {
            case 2: return run_gemv<2, 1>(bits, sc, rows, cols, x, batch, y, s);
            case 3: return run_gemv<3, 1>(bits, sc, rows, cols, x, batch, y, s);
            default: return run_gemv<4, 1>(bits, sc, rows, cols, x, batch, y, s);
        }
    }
    switch (K) {
        case 2: return run_gemv<2, 2>(bits, sc, rows, cols, x, batch, y, s);
        case 3: return run_gemv<3, 2>(bits, sc, rows, cols, x, batch, y, s);
        default: return run_gemv<4, 2>(bits, sc, rows, cols, x, batch, y, s);
    }
}

TQ_API size_t moe_trellis_workspace_size(const tq_moe_layer *layer, int T, int k) {
    if (validate_layer(layer) != TQ_OK || T < 0 || k < 1) return 0;
    return workspace_bytes(layer, T, k);
}

int moe_validate_call(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                      const int32_t *perm, const int32_t *active_ids, const int32_t *n_active, int T,
                      int k, float *y_perm, void *ws, size_t ws_bytes) {
    int st = validate_layer(layer);
    if (st) return st;
    if (T < 0 || k < 1 || k > layer->E) return TQ_ERR_INVALID_ARG;
    if ((long long)T * k > (1ll << 30)) return TQ_ERR_UNSUPPORTED;
    if (T == 0) return TQ_OK;
    if (!x_rot || !offsets || !perm || !active_ids || !n_active || !y_perm) return TQ_ERR_INVALID_ARG;
    if (!aligned16(x_rot) || !aligned16(y_perm)) return TQ_ERR_ALIGNMENT;
    if (!ws || ws_bytes < workspace_bytes(layer, T, k)) return TQ_ERR_WORKSPACE;
    if (!aligned16(ws)) return TQ_ERR_ALIGNMENT;
    return TQ_OK;
}

TQ_API int moe_trellis_gemv(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                            const int32_t *perm, const int32_t *active_ids, const int32_t *n_active, int T,
                            int k, float *y_perm, void *ws, size_t ws_bytes, tq_stream stream) {
    int st = moe_validate_call(layer, x_rot, offsets, perm, active_ids, n_active, T, k, y_perm, ws, ws_bytes);
    if (st || T == 0) return st;
    const __half *x = reinterpret_cast<const __half *>(x_rot);
    cudaStream_t s = (cudaStream_t)stream;
    if (T <= 8) return run_moe_gemv<1>(layer, x, offsets, perm, active_ids, n_active, T, k, y_perm, ws, s);
    return run_moe_gemv<2>(layer, x, offsets, perm, active_ids, n_active, T, k, y_perm, ws, s);
}
