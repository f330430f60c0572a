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

// Subnormal planes: D = 2^-24 * sum_j t_j x_j, so sum_j c_j x_j = 2^24 D - 255 sum_j x_j.
__device__ __forceinline__ float finish_sub(float d, float sx, float scale) {
    return scale * kKappa * fmaf(16777216.0f, d, -255.0f * sx);
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
    extern __shared__ __align__(128) unsigned char smem_raw[];
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
    int group, index;             // width group and position inside it
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
    r.group = gi;
    r.index = idx;
    r.gate = G.gate + (size_t)idx * words_proj;
    r.up = G.up + (size_t)idx * words_proj;
    r.down = G.down + (size_t)idx * words_proj;
    r.s_gate = reinterpret_cast<const __half *>(G.s_gate) + (size_t)idx * L.F;
    r.s_up = reinterpret_cast<const __half *>(G.s_up) + (size_t)idx * L.F;
    r.s_down = reinterpret_cast<const __half *>(G.s_down) + (size_t)idx * L.D;
    return true;
}

// ----------------------------------------------------------------------------- MoE items
//
// MoE GEMV work item = one CTA of kItemWarps warps: (active expert, 8 strips of 16
// rows, 8 of the expert's routes).  The warps split the column tiles into contiguous
// ranges; each streams its range of the 8 strips through its own ring of shared-memory
// stages filled by bulk copies (lanes 0..7 copy one strip each, completing on one
// mbarrier per stage; consumers poll with a bound), and the warps' MMA partial sums
// are added in shared memory in a fixed order at the end of the item.
//
// Per weight: one funnel shift brings the window to bit 0 (none for windows that start
// a word), one integer multiply by 0x3A2F0000 leaves the T16 product's bytes lo, hi in
// bytes 2 and 3 with zeros below, and one PRMT pairs the lo (or hi) bytes of two
// weights with zero bytes: fp16 subnormals lo * 2^-24 and hi * 2^-24, exact operands.
// The MMA accumulates D = 2^-24 * sum_j t_j x_j in fp32 (no offset to cancel).

constexpr int kItemWarps = 4;
constexpr int kItemThreads = kItemWarps * 32;
constexpr int kStages = 2;
constexpr int kSlotBytes = 576;               // per strip per stage: >= 8*64, 5*96, 4*128 B,
                                              // 64 B pad so 2 strips share no bank in a phase
constexpr int kStageBytes = 8 * kSlotBytes;

template <int K>
constexpr int tiles_per_stage() { return K == 2 ? 8 : (K == 3 ? 5 : 4); }

// A warp's ring: its stage buffers and one mbarrier per stage.  The barriers live in a
// region of their own (ItemSmem::bar) that nothing else ever writes: an mbarrier's
// memory must not be reused by ordinary stores while the barrier is initialised.
struct WarpRing {
    unsigned char (*buf)[kStageBytes];
    uint64_t *bar;
};

struct __align__(128) ItemSmem {
    unsigned char buf[kItemWarps][kStages][kStageBytes];
    uint64_t bar[kItemWarps][kStages];
};

// T16 product of the window at compile-time bit offset O of the lane's span, in the
// high half of the result (low half zero): bytes [0, 0, lo, hi].
template <int O, int NS>
__device__ __forceinline__ uint32_t t16_product_hi(const uint32_t (&v)[NS]) {
    constexpr int wi = O >> 5, sh = O & 31;
    uint32_t bottom;
    if constexpr (sh == 0) bottom = v[wi];
    else bottom = funnel_r(v[wi], v[wi + 1], sh);
    return bottom * (kT16Mult << 16);
}

template <int K, int P>
__device__ __forceinline__ void tile_pairs_sub(const uint32_t (&v)[2 * K + 1], uint2 xb, Acc<1> &acc) {
    if constexpr (P < 8) {
        constexpr int r0 = P, r1 = P + 8;
        const uint32_t R00 = t16_product_hi<0 * 16 * K + K * r0>(v);
        const uint32_t R01 = t16_product_hi<1 * 16 * K + K * r0>(v);
        const uint32_t R02 = t16_product_hi<2 * 16 * K + K * r0>(v);
        const uint32_t R03 = t16_product_hi<3 * 16 * K + K * r0>(v);
        const uint32_t R10 = t16_product_hi<0 * 16 * K + K * r1>(v);
        const uint32_t R11 = t16_product_hi<1 * 16 * K + K * r1>(v);
        const uint32_t R12 = t16_product_hi<2 * 16 * K + K * r1>(v);
        const uint32_t R13 = t16_product_hi<3 * 16 * K + K * r1>(v);
        mma_f16_16816(acc.d[P][0], prmt(R00, R01, kSelLo), prmt(R10, R11, kSelLo), prmt(R02, R03, kSelLo),
                      prmt(R12, R13, kSelLo), xb.x, xb.y);
        mma_f16_16816(acc.d[P][0], prmt(R00, R01, kSelHi), prmt(R10, R11, kSelHi), prmt(R02, R03, kSelHi),
                      prmt(R12, R13, kSelHi), xb.x, xb.y);
        tile_pairs_sub<K, P + 1>(v, xb, acc);
    }
}

__device__ __forceinline__ void ring_init(const WarpRing &ring) {
    const int lane = threadIdx.x & 31;
    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&ring.bar[s], 1);
        fence_barrier_init();
    }
    __syncwarp();
}

// Issue chunk c (tiles [j0 + c*S, ...), at most `je` exclusive) of the 8 strips into
// stage st.  strip_lane: base of the strip this lane copies (lanes 0..7).
template <int K>
__device__ __forceinline__ void ring_issue(const WarpRing &ring, int st, int c, int j0, int je,
                                           const uint32_t *strip_lane) {
    constexpr int S = tiles_per_stage<K>();
    constexpr int TB = 32 * K;  // bytes per tile
    const int lane = threadIdx.x & 31;
    const int jb = j0 + c * S;
    const int nt = min(S, je - jb);
    if (lane == 0) {
        fence_proxy_async();
        mbar_arrive_expect_tx(&ring.bar[st], 8u * nt * TB);
    }
    __syncwarp();
    if (lane < 8) bulk_g2s(ring.buf[st] + lane * kSlotBytes, strip_lane + (size_t)jb * (8 * K), nt * TB, &ring.bar[st]);
}

// Stream tiles [j0, je) of the 8 strips against the lane's token row xr (fp16 or null).
// Returns false, after draining its copies, if a bounded wait gave up.
template <int K>
__device__ __forceinline__ bool stream_range(const WarpRing &ring, uint32_t &parity, int j0, int je,
                                          const uint32_t *strip_lane, const __half *xr, Acc<1> &acc) {
    constexpr int S = tiles_per_stage<K>();
    constexpr int TB = 32 * K;
    const int lane = threadIdx.x & 31, gq = lane >> 2, t4 = lane & 3;
    const int n_chunks = (je - j0 + S - 1) / S;
    for (int c = 0; c < min(kStages, n_chunks); ++c) ring_issue<K>(ring, c, c, j0, je, strip_lane);
    uint2 xn = (xr && j0 < je) ? __ldg(reinterpret_cast<const uint2 *>(xr + 16 * j0 + 4 * t4)) : make_uint2(0u, 0u);
    for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kStages;
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&ring.bar[st], (parity >> st) & 1u));
        parity ^= 1u << st;
        if (!ok) {
            for (int d = c + 1; d < min(c + kStages, n_chunks); ++d) {
                const int sd = d % kStages;
                mbar_wait_bounded(&ring.bar[sd], (parity >> sd) & 1u);
                parity ^= 1u << sd;
            }
            return false;
        }
        const int jb = j0 + c * S;
        const int nt = min(S, je - jb);
        const unsigned char *slot = ring.buf[st] + gq * kSlotBytes;
#pragma unroll 1
        for (int t = 0; t < nt; ++t) {
            const unsigned char *tile = slot + t * TB;
            uint32_t v[2 * K + 1];
            if constexpr (K == 2) {
                uint4 a = *reinterpret_cast<const uint4 *>(tile + 16 * t4);
                v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            } else if constexpr (K == 3) {
                const uint2 *q = reinterpret_cast<const uint2 *>(tile + 24 * t4);
                uint2 a = q[0], b = q[1], d = q[2];
                v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y; v[4] = d.x; v[5] = d.y;
            } else {
                const uint4 *q = reinterpret_cast<const uint4 *>(tile + 32 * t4);
                uint4 a = q[0], b = q[1];
                v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
                v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
            }
            v[2 * K] = *reinterpret_cast<const uint32_t *>(tile + 8 * K * ((t4 + 1) & 3));
            const uint2 x = xn;
            const int jn = jb + t + 1;
            if (xr && jn < je) xn = __ldg(reinterpret_cast<const uint2 *>(xr + 16 * jn + 4 * t4));
            tile_pairs_sub<K, 0>(v, x, acc);
            mma_f16_16816(acc.s[0], kOneH2, kOneH2, kOneH2, kOneH2, x.x, x.y);
        }
        __syncwarp();
        if (c + kStages < n_chunks) ring_issue<K>(ring, st, c + kStages, j0, je, strip_lane);
    }
    return true;
}

// Shared-memory partials of the CTA's warps; aliases the stage buffers (never the
// barriers) once every warp has consumed its last stage.
struct ItemRed {
    float d[kItemWarps][8][16][8];   // [warp][strip][row][token]
    float s[kItemWarps][8];          // [warp][token]
};
static_assert(sizeof(ItemRed) <= sizeof(ItemSmem::buf), "reduction buffer must fit in the stage buffers");

// GATEUP: item = (active expert, 64 intermediate rows: strips 0..3 of gate, 0..3 of up),
//         out = h [routes][F] fp32, h = silu(gate x') * (up x').
// !GATEUP: item = (active expert, 128 output rows), xsrc = h' [routes][F] fp16,
//          out = y [routes][D] fp32.
template <bool GATEUP>
__global__ void __launch_bounds__(kItemThreads, 5)
    moe_gemv_items_kernel(const tq_moe_layer L, const __half *__restrict__ xsrc,
                          const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm,
                          const int32_t *__restrict__ active_ids, const int32_t *__restrict__ n_active_p,
                          int k, int n_routes, float *__restrict__ out) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    ItemSmem &sm_items = *reinterpret_cast<ItemSmem *>(smem_raw);
    ItemRed &red = *reinterpret_cast<ItemRed *>(smem_raw);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gq = lane >> 2, t4 = lane & 3;
    const int per_expert = GATEUP ? L.F / 64 : L.D / 128;
    const int item = blockIdx.x;
    if (item >= *n_active_p * per_expert) return;
    const int a = item / per_expert, sub = item % per_expert;
    const int e = active_ids[a];
    ExpertRef ex;
    if (!expert_ref(L, e, ex)) {
        if (threadIdx.x == 0) raise_flag(1);
        return;
    }
    const WarpRing ring{sm_items.buf[warp], sm_items.bar[warp]};
    ring_init(ring);
    uint32_t parity = 0;

    const int r0 = offsets[e], ne = offsets[e + 1] - r0;
    const int tiles = GATEUP ? L.D / 16 : L.F / 16;
    int jb, je;
    split_range(tiles, warp, kItemWarps, jb, je);
    const int cs = lane & 7;
    const uint32_t *strip_lane;
    if (GATEUP)
        strip_lane = (cs < 4 ? ex.gate : ex.up) + (size_t)(sub * 4 + (cs & 3)) * tiles * (8 * ex.K);
    else
        strip_lane = ex.down + (size_t)(sub * 8 + cs) * tiles * (8 * ex.K);

    for (int tb = 0; tb < ne; tb += 8) {
        const int tt = tb + gq;
        const __half *xr = nullptr;
        if (tt < ne) {
            if (GATEUP) {
                const int pr = perm[r0 + tt];
                if (pr >= 0 && pr < n_routes) xr = xsrc + (size_t)(pr / k) * L.D;
            } else {
                xr = xsrc + (size_t)(r0 + tt) * L.F;
            }
        }
        Acc<1> acc;
        zero(acc);
        bool ok;
        if (ex.K == 2) ok = stream_range<2>(ring, parity, jb, je, strip_lane, xr, acc);
        else if (ex.K == 3) ok = stream_range<3>(ring, parity, jb, je, strip_lane, xr, acc);
        else ok = stream_range<4>(ring, parity, jb, je, strip_lane, xr, acc);
        ok = __syncthreads_and(ok);
        if (!ok) return;   // every warp drained its copies; the item is left unwritten
        // partials -> shared memory (the rings are idle now)
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            red.d[warp][gq][p][2 * t4] = acc.d[p][0][0];
            red.d[warp][gq][p][2 * t4 + 1] = acc.d[p][0][1];
            red.d[warp][gq][p + 8][2 * t4] = acc.d[p][0][2];
            red.d[warp][gq][p + 8][2 * t4 + 1] = acc.d[p][0][3];
        }
        if (gq == 0) {
            red.s[warp][2 * t4] = acc.s[0][0];
            red.s[warp][2 * t4 + 1] = acc.s[0][1];
        }
        __syncthreads();
        if (GATEUP) {
            for (int i = threadIdx.x; i < 4 * 16 * 8; i += kItemThreads) {
                const int tok = i & 7, row = (i >> 3) & 15, st = i >> 7;
                const int t2 = tb + tok;
                if (t2 >= ne) continue;
                float dg = 0.f, du = 0.f, sx = 0.f;
#pragma unroll
                for (int w = 0; w < kItemWarps; ++w) {
                    dg += red.d[w][st][row][tok];
                    du += red.d[w][st + 4][row][tok];
                    sx += red.s[w][tok];
                }
                const int f = (sub * 4 + st) * 16 + row;
                const float gv = finish_sub(dg, sx, __half2float(ex.s_gate[f]));
                const float uv = finish_sub(du, sx, __half2float(ex.s_up[f]));
                out[(size_t)(r0 + t2) * L.F + f] = silu_f32(gv) * uv;
            }
        } else {
            for (int i = threadIdx.x; i < 8 * 16 * 8; i += kItemThreads) {
                const int tok = i & 7, row = (i >> 3) & 15, st = i >> 7;
                const int t2 = tb + tok;
                if (t2 >= ne) continue;
                float dd = 0.f, sx = 0.f;
#pragma unroll
                for (int w = 0; w < kItemWarps; ++w) {
                    dd += red.d[w][st][row][tok];
                    sx += red.s[w][tok];
                }
                const int d = (sub * 8 + st) * 16 + row;
                out[(size_t)(r0 + t2) * L.D + d] = finish_sub(dd, sx, __half2float(ex.s_down[d]));
            }
        }
        __syncthreads();   // the rings are reused by the next pass
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

int run_moe_gemv(const tq_moe_layer *L, const __half *x_rot, const int32_t *offsets, const int32_t *perm,
                 const int32_t *active_ids, const int32_t *n_active, int T, int k, float *y_perm,
                 void *ws, cudaStream_t s) {
    const size_t smem = sizeof(ItemSmem);
    static bool configured = false;
    if (!configured) {
        if (set_smem(moe_gemv_items_kernel<true>, smem) || set_smem(moe_gemv_items_kernel<false>, smem))
            return TQ_ERR_CUDA;
        configured = true;
    }
    const int routes = T * k;
    float *h = reinterpret_cast<float *>(ws);
    __half *h_rot = reinterpret_cast<__half *>(reinterpret_cast<char *>(ws) +
                                               align256((size_t)routes * L->F * sizeof(float)));
    const int max_active = min(L->E, routes);
    const int gu_items = max_active * (L->F / 64);
    const int dn_items = max_active * (L->D / 128);
    {
        LaunchScope ls(s, kStageGemvGateUp);
        moe_gemv_items_kernel<true><<<gu_items, kItemThreads, smem, s>>>(*L, x_rot, offsets, perm, active_ids,
                                                                          n_active, k, routes, h);
    }
    int st = launch_status();
    if (st) return st;
    st = launch_hadamard128(h, TQ_DTYPE_F32, routes, L->F, h_rot, s, kStageRotateH);
    if (st) return st;
    LaunchScope ls(s, kStageGemvDown);
    moe_gemv_items_kernel<false><<<dn_items, kItemThreads, smem, s>>>(*L, h_rot, offsets, perm, active_ids,
                                                                       n_active, k, routes, y_perm);
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

namespace tq {
size_t gemm_workspace_bytes(const tq_moe_layer *L, int T, int k);
}

TQ_API size_t moe_trellis_workspace_size(const tq_moe_layer *layer, int T, int k) {
    if (validate_layer(layer) != TQ_OK || T < 0 || k < 1) return 0;
    const size_t gemv = workspace_bytes(layer, T, k), gemm = tq::gemm_workspace_bytes(layer, T, k);
    return gemv > gemm ? gemv : gemm;
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
    return run_moe_gemv(layer, x, offsets, perm, active_ids, n_active, T, k, y_perm, ws, s);
}
