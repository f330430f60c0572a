// Decode-fused GEMV for T16 trellis-coded matrices: single projection (trellis_gemv)
// and the routed experts of a MoE layer for decode-sized batches (moe_trellis_gemv).
//
// Method: "DeepSeek-V4.1-Flash-1017 · dsx T16", "How T16 works" -- item 1 (T16: the
// 16-bit window times 0x3A2F mod 2^16, plus the product's two bytes), item 2
// (column-major 16x16 tiles), item 4 (per-output scales); gate/up/SiLU/down of the
// routed experts with fused gate/up post-processing ("October 25 runtime checkpoint").
//
// Decode in registers, contraction on the tensor cores with integer MMAs
// (mma.sync m16n8k32, u8 weights x s8 activations -> s32, exact):
//   * Activations enter as 16-bit fixed point, one power of two per row:
//     x_q = round(x / 2^e), |x_q| <= 32639, split into two signed bytes
//     x_q = 256 xh + xl (xl in [-128, 127]).  quantize_rows_kernel writes each byte
//     twice into a half-word (one row of xh half-words, one of xl half-words) and e
//     and sum_j x_q of every row.  A row whose rounding step is coarse for its mass
//     (2^(e-1) * cols > 2^-12 * sum_j |x_j|: a few elements dominate) also gets a second
//     word, the residual x - x_q 2^e as 16-bit fixed point at 2^(e-15), so such a row is
//     32-bit fixed point; its two words take two MMA column pairs ("slots").
//   * A warp walks 8 strips (16 output rows each): lane group g = lane/4 owns strip g
//     and lane t = lane%4 owns columns 4t..4t+3 of each tile, so every lane decodes the
//     same tile-relative bit offsets (compile-time shifts).
//   * Window -> A operand: one funnel shift brings the window to bit 0 (none when it
//     starts a word) and one integer multiply by 0x3A2F0000 leaves bytes [0, 0, lo, hi],
//     lo/hi the two bytes of (window * 0x3A2F) mod 2^16.  One A register is one weight
//     spread over 4 k-slots; its two zero slots meet whatever the activation word holds
//     there, so the MMA adds (lo + hi) * x = t * x with no byte shuffling.
//   * The MMA's 8 columns are 4 slots x 2 limbs (column 2r: slot r's xh, 2r+1: its
//     xl); a slot holds one word of one route.  |partial sums| <= 510 * 128 * cols <
//     2^31 for cols <= 16384.
//   * Epilogue, in double: y = s * 2^-12 * 2^e * (256 H + L - 255 sum_j x_q), H and L
//     the two limb sums (sum_j c_j x_j = sum_j t_j x_j - 255 sum_j x_j), plus
//     2^(e-15) * (256 H' + L' - 255 sum_j r_q) from the residual slot of a two-word row.
//   * Bit streams reach shared memory by bulk copies into a per-warp ring of stages
//     (one mbarrier per stage, bounded waits); activations come from L2, one tile
//     ahead.
#include "tq_common.cuh"

namespace tq {

constexpr int kMaxCols = 16384;        // keeps every int32 partial sum in range
constexpr int kQMax = 32639;           // 127 * 256 + 127: both bytes stay signed
constexpr int kResShift = 15;          // residual word scale: 2^(e - 15)
constexpr int kResBudgetLog2 = 12;     // second word when 2^(e-1) * cols > 2^-12 * sum |x|

// Fixed-point activation row: x ~ x_q 2^e (+ r_q 2^(e - kResShift) when res != 0).
// Planes of a row in memory: [0] xh half-words, [1] xl, [2] rh, [3] rl (cols each).
struct __align__(16) RowQ {
    int e;        // power of two of the main word
    int sum;      // sum_j x_q
    int res;      // 1: the row carries the residual word
    int rsum;     // sum_j r_q
};
constexpr int kItemWarps = 4;
constexpr int kItemThreads = kItemWarps * 32;
constexpr int kStages = 2;
constexpr int kSlotBytes = 576;        // per strip per stage: >= 8*64, 5*96, 4*128 B,
                                       // 64 B pad so 2 strips share no bank in a phase
constexpr int kStageBytes = 8 * kSlotBytes;

template <int K>
constexpr int tiles_per_stage() { return K == 2 ? 8 : (K == 3 ? 5 : 4); }

__device__ __forceinline__ void imma_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

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

// Integer accumulators of NB blocks of 4 routes: [row pair P][block][fragment];
// fragment 0/1 = (row P, route t, limb h/l), 2/3 = (row P + 8, ...).
template <int NB>
struct AccI {
    int d[8][NB][4];
};

template <int NB>
__device__ __forceinline__ void zero(AccI<NB> &acc) {
#pragma unroll
    for (int p = 0; p < 8; ++p)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc.d[p][b][i] = 0;
}

// Rows P and P + 8 of the lane's tile against its 4 columns: 8 windows, 2 MMAs per
// block (columns 4t, 4t+1 as k-slot groups t, 4+t; then columns 4t+2, 4t+3).
template <int K, int NB, int P>
__device__ __forceinline__ void tile_rows(const uint32_t (&v)[2 * K + 1], const uint4 (&xb)[NB], AccI<NB> &acc) {
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
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            imma_16832(acc.d[P][b], R00, R10, R01, R11, xb[b].x, xb[b].y);
            imma_16832(acc.d[P][b], R02, R12, R03, R13, xb[b].z, xb[b].w);
        }
        tile_rows<K, NB, P + 1>(v, xb, acc);
    }
}

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

// Activation half-words of the lane's 4 columns of tile j (null row: zeros): each
// 16-bit value holds one signed byte twice, so a 32-bit word [x_c x_c x_c+1 x_c+1]
// is the B operand of column c+1 (bytes 2, 3) and, shifted left by 16, of column c.
// FRESH: the rows were written earlier in this same launch (published by a release and
// picked up by a gpu-scope acquire before the read), so they take plain coherent loads,
// which may hit L1, instead of the read-only path.
__device__ __forceinline__ uint2 ld_weak_v2(const uint2 *p) {
    uint2 v;
    asm volatile("ld.global.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

template <bool FRESH = false>
__device__ __forceinline__ uint2 x_halves(const uint16_t *xw, int j, int t4) {
    if (!xw) return make_uint2(0u, 0u);
    const uint2 *p = reinterpret_cast<const uint2 *>(xw + 16 * j + 4 * t4);
    return FRESH ? ld_weak_v2(p) : __ldg(p);
}

// Stream tiles [j0, je) of the 8 strips against the lane's activation rows xw[b] (the
// lane's limb of route 4b + g/2 of the pass, or null); activations are loaded one tile
// ahead.  Returns false, after draining its copies, if a bounded wait gave up.
template <int K, int NB, bool FRESH = false>
__device__ __forceinline__ bool stream_range(const WarpRing &ring, uint32_t &parity, int j0, int je,
                                             const uint32_t *strip_lane, const uint16_t *const (&xw)[NB],
                                             AccI<NB> &acc) {
    constexpr int S = tiles_per_stage<K>();
    constexpr int TB = 32 * K;
    const int lane = threadIdx.x & 31, gq = lane >> 2, t4 = lane & 3;
    const int n_chunks = (je - j0 + S - 1) / S;
    for (int c = 0; c < min(kStages, n_chunks); ++c) ring_issue<K>(ring, c, c, j0, je, strip_lane);
    uint2 xn[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) xn[b] = j0 < je ? x_halves<FRESH>(xw[b], j0, t4) : make_uint2(0u, 0u);
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
            // word after the lane's quarter: the next quarter's first (tail-biting)
            v[2 * K] = *reinterpret_cast<const uint32_t *>(tile + 8 * K * ((t4 + 1) & 3));
            uint4 x[NB];
#pragma unroll
            for (int b = 0; b < NB; ++b) x[b] = make_uint4(xn[b].x << 16, xn[b].x, xn[b].y << 16, xn[b].y);
            const int jn = jb + t + 1;
            if (jn < je) {
#pragma unroll
                for (int b = 0; b < NB; ++b) xn[b] = x_halves<FRESH>(xw[b], jn, t4);
            }
            tile_rows<K, NB, 0>(v, x, acc);
        }
        __syncwarp();
        if (c + kStages < n_chunks) ring_issue<K>(ring, st, c + kStages, j0, je, strip_lane);
    }
    return true;
}

template <int NB, bool FRESH = false>
__device__ __forceinline__ bool stream_any(int K, const WarpRing &ring, uint32_t &parity, int j0, int je,
                                           const uint32_t *strip_lane, const uint16_t *const (&xw)[NB],
                                           AccI<NB> &acc) {
    if (K == 2) return stream_range<2, NB, FRESH>(ring, parity, j0, je, strip_lane, xw, acc);
    if (K == 3) return stream_range<3, NB, FRESH>(ring, parity, j0, je, strip_lane, xw, acc);
    return stream_range<4, NB, FRESH>(ring, parity, j0, je, strip_lane, xw, acc);
}

// Shared-memory partials of the CTA's warps; aliases the stage buffers (never the
// barriers) once every warp has consumed its last stage.
template <int NB>
struct ItemRed {
    int d[kItemWarps][8][16][4 * NB][2];   // [warp][strip][row][route][limb]
};
static_assert(sizeof(ItemRed<2>) <= sizeof(ItemSmem::buf), "reduction buffer must fit in the stage buffers");

template <int NB>
__device__ __forceinline__ void store_partials(const AccI<NB> &acc, ItemRed<NB> &red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gq = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int p = 0; p < 8; ++p)
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            *reinterpret_cast<int2 *>(red.d[warp][gq][p][4 * b + t4]) = make_int2(acc.d[p][b][0], acc.d[p][b][1]);
            *reinterpret_cast<int2 *>(red.d[warp][gq][p + 8][4 * b + t4]) = make_int2(acc.d[p][b][2], acc.d[p][b][3]);
        }
}

// Sum over warps in fixed order (exact): limb sums of (strip, row, route).
template <int NB>
__device__ __forceinline__ int2 red_sum(const ItemRed<NB> &red, int strip, int row, int route) {
    int h = 0, l = 0;
#pragma unroll
    for (int w = 0; w < kItemWarps; ++w) {
        h += red.d[w][strip][row][route][0];
        l += red.d[w][strip][row][route][1];
    }
    return make_int2(h, l);
}

// y = s * 2^-12 * 2^e * (256 H + L - 255 sum x_q), formed in double (the integer part
// and the scale are exact doubles, so the result is rounded once to double and once to
// float).  A two-word row adds its residual sums (H2, L2) at 2^-15 of the main word's
// scale: 2^15 a + a2 stays below 2^53 for cols <= 16384, so it is exact too.
__device__ __forceinline__ float finish_q(int H, int L, const RowQ &q, float scale, int H2 = 0, int L2 = 0) {
    double a = 256.0 * (double)H + (double)L - 255.0 * (double)q.sum;
    int e = q.e;
    if (q.res) {
        a = a * (double)(1 << kResShift) + (256.0 * (double)H2 + (double)L2 - 255.0 * (double)q.rsum);
        e -= kResShift;
    }
    return (float)(a * ldexp((double)scale * (double)kKappa, e));
}

__device__ __forceinline__ void split_range(int n, int part, int parts, int &b, int &e) {
    const int per = (n + parts - 1) / parts;
    b = min(n, part * per);
    e = min(n, b + per);
}

// ------------------------------------------------------------------ activation rows
//
// One CTA of 8 warps per row of `cols` values (a multiple of 128): take the row from
// its source (optionally rotating every 128-chunk with fwht128_warp, the hadamard128
// transform), take max |v| and sum |v| over the row, pick e with max / 2^e <= 32639
// (e = ilogb(max) - 14, one more if the mantissa is too large), and write
// x_q = rint(v / 2^e) as its two signed bytes, each held twice in a half-word:
// xq[row][0][col] = xh * 0x0101, xq[row][1][col] = xl * 0x0101.  When
// 2^(e-1) * cols > 2^-12 * sum |v| the row also gets its residual word
// r_q = rint((v - x_q 2^e) / 2^(e-15)) (|r_q| <= 2^14; v - x_q 2^e is exact in fp32) in
// planes 2 and 3.  meta[row] = (e, sum x_q, residual flag, sum r_q).  A warp keeps its
// first KEPT chunks in registers between the two passes; further chunks (rows longer
// than KEPT * 128 * WARPS) are read again in the second pass.

// Plain rows x[row][cols].
template <typename T>
struct RowSrc {
    const T *x;
    int cols;
    __device__ __forceinline__ void load(int row, int c, int lane, float (&v)[4]) const {
        const float4 f = load4<T>(x + (size_t)row * cols + (size_t)c * 128 + 4 * lane);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    }
};

// SwiGLU of the gate/up GEMV's column-split partial sums: h = silu(sum_s g_s) * sum_s u_s
// from gu[row][s][0][cols] (gate) and gu[row][s][1][cols] (up), summed in split order.
// sign_gu (optional): the output side of the two-sided transform, applied to g and u
// before the SwiGLU: g = sign_gu * rotate(g), u likewise.
__device__ __forceinline__ void swiglu_finish(float4 g, float4 u, const int8_t *sign_gu, int c, int lane,
                                              float (&v)[4]) {
    float gv[4] = {g.x, g.y, g.z, g.w}, uv[4] = {u.x, u.y, u.z, u.w};
    if (sign_gu) {
        fwht128_warp(gv, lane);
        fwht128_warp(uv, lane);
        const char4 sg = *reinterpret_cast<const char4 *>(sign_gu + c * 128 + 4 * lane);
        const float s4[4] = {(float)sg.x, (float)sg.y, (float)sg.z, (float)sg.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            gv[i] *= s4[i];
            uv[i] *= s4[i];
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = silu_f32(gv[i]) * uv[i];
}

// The partials read from global memory through L2 (the h' quantisation launch).
struct SwigluSrc {
    const float *gu;
    int cols, splits;
    const int8_t *sign_gu;
    __device__ __forceinline__ void load(int row, int c, int lane, float (&v)[4]) const {
        const float *p = gu + (size_t)row * splits * 2 * cols + (size_t)c * 128 + 4 * lane;
        float4 g = __ldcg(reinterpret_cast<const float4 *>(p)), u = __ldcg(reinterpret_cast<const float4 *>(p + cols));
        for (int sp = 1; sp < splits; ++sp) {
            const float4 g2 = __ldcg(reinterpret_cast<const float4 *>(p + (size_t)sp * 2 * cols));
            const float4 u2 = __ldcg(reinterpret_cast<const float4 *>(p + (size_t)sp * 2 * cols + cols));
            g.x += g2.x; g.y += g2.y; g.z += g2.z; g.w += g2.w;
            u.x += u2.x; u.y += u2.y; u.z += u2.z; u.w += u2.w;
        }
        swiglu_finish(g, u, sign_gu, c, lane, v);
    }
};

// The same inside the fused kernel.  staged: gu is one route's [s][2][cols] already in
// shared memory (stage_row_async; the row argument is ignored); otherwise the partials
// are read from global memory through L2 (they were written by other CTAs of the same
// launch).
struct SwigluFusedSrc {
    const float *gu;
    int cols, splits;
    const int8_t *sign_gu;
    bool staged;
    __device__ __forceinline__ float4 ld(const float *p) const {
        return staged ? *reinterpret_cast<const float4 *>(p) : __ldcg(reinterpret_cast<const float4 *>(p));
    }
    __device__ __forceinline__ void load(int row, int c, int lane, float (&v)[4]) const {
        const float *p = gu + (staged ? 0 : (size_t)row * splits * 2 * cols) + (size_t)c * 128 + 4 * lane;
        float4 g = ld(p), u = ld(p + cols);
        for (int sp = 1; sp < splits; ++sp) {
            const float4 g2 = ld(p + (size_t)sp * 2 * cols), u2 = ld(p + (size_t)sp * 2 * cols + cols);
            g.x += g2.x; g.y += g2.y; g.z += g2.z; g.w += g2.w;
            u.x += u2.x; u.y += u2.y; u.z += u2.z; u.w += u2.w;
        }
        swiglu_finish(g, u, sign_gu, c, lane, v);
    }
};

// Rows whose values are final (already rotated): h[c * 128 + 4 * lane ...] through a
// generic pointer (shared or global memory); the row argument is ignored.
struct FinalRowSrc {
    const float *h;
    __device__ __forceinline__ void load(int, int c, int lane, float (&v)[4]) const {
        const float4 f = *reinterpret_cast<const float4 *>(h + (size_t)c * 128 + 4 * lane);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    }
};

// One route's split partials (bytes, a multiple of 16) copied from global memory into
// shared memory with 16-byte cp.async copies through L2, all in flight at once; returns
// after the CTA's copies have landed.
__device__ __forceinline__ void stage_row_async(unsigned char *dst, const float *src, int bytes) {
    const uint32_t d = smem_u32(dst);
    const char *g = reinterpret_cast<const char *>(src);
    for (int o = threadIdx.x * 16; o < bytes; o += kItemThreads * 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d + o), "l"(g + o) : "memory");
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncthreads();
}

// One row quantised by the whole CTA (WARPS warps); the s_* arrays hold WARPS entries.
// KEPT: 128-value chunks per warp kept in registers between the two passes.
template <int WARPS, typename Src, bool ROTATE, int KEPT>
__device__ __forceinline__ void quantize_row(const Src &src, int row, int cols, const int8_t *__restrict__ signs,
                                             uint16_t *__restrict__ xq, RowQ *__restrict__ meta, float *s_max,
                                             float *s_l1, int *s_sum, int *s_rsum) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int chunks = cols / 128;
    auto load = [&](int c, float (&v)[4]) {
        src.load(row, c, lane, v);
        if constexpr (ROTATE) {
            if (signs) {   // input side of the two-sided transform: rotate(signs * v)
                const char4 sg = *reinterpret_cast<const char4 *>(signs + c * 128 + 4 * lane);
                v[0] *= sg.x; v[1] *= sg.y; v[2] *= sg.z; v[3] *= sg.w;
            }
            fwht128_warp(v, lane);
        }
    };
    // pass 1: max |v| and sum |v|, chunks in increasing order (the first KEPT of
    // the warp's chunks stay in registers)
    float m = 0.f, l1 = 0.f;
    float kept[KEPT > 0 ? KEPT : 1][4];
#pragma unroll
    for (int j = 0; j < KEPT; ++j) {
        const int c = warp + j * WARPS;
        if (c < chunks) {
            load(c, kept[j]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                m = fmaxf(m, fabsf(kept[j][i]));
                l1 += fabsf(kept[j][i]);
            }
        }
    }
    for (int c = warp + KEPT * WARPS; c < chunks; c += WARPS) {
        float v[4];
        load(c, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            m = fmaxf(m, fabsf(v[i]));
            l1 += fabsf(v[i]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    if (lane == 0) {
        s_max[warp] = m;
        s_l1[warp] = l1;
    }
    __syncthreads();
    m = s_max[0];
    l1 = s_l1[0];
#pragma unroll
    for (int w = 1; w < WARPS; ++w) {
        m = fmaxf(m, s_max[w]);
        l1 += s_l1[w];
    }
    int e = 0;
    if (m > 0.f) {                   // a NaN or infinite max is not supported
        e = ilogbf(m) - 14;
        if (ldexpf(m, -e) > (float)kQMax) ++e;
    }
    // second word when the rounding step, summed over the row, exceeds 2^-12 of its mass
    const bool res = m > 0.f && ldexpf((float)cols, e - 1) > ldexpf(l1, -kResBudgetLog2);
    uint16_t *qh = xq + (size_t)row * 4 * cols, *ql = qh + cols, *rh = ql + cols, *rl = rh + cols;
    int sum = 0, rsum = 0;
    auto quantize_chunk = [&](int c, const float (&v)[4]) {
        uint32_t wh[4], wl[4], vh[4], vl[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int q = __float2int_rn(ldexpf(v[i], -e));
            q = max(-kQMax, min(kQMax, q));
            sum += q;
            const int lo = ((q + 128) & 255) - 128;
            const int hi = (q - lo) >> 8;
            wh[i] = (uint32_t)(hi & 255) * 0x0101u;
            wl[i] = (uint32_t)(lo & 255) * 0x0101u;
            if (res) {
                const float r = __fsub_rn(v[i], ldexpf((float)q, e));   // exact
                int rq = __float2int_rn(ldexpf(r, kResShift - e));
                rq = max(-kQMax, min(kQMax, rq));
                rsum += rq;
                const int rlo = ((rq + 128) & 255) - 128;
                const int rhi = (rq - rlo) >> 8;
                vh[i] = (uint32_t)(rhi & 255) * 0x0101u;
                vl[i] = (uint32_t)(rlo & 255) * 0x0101u;
            }
        }
        const size_t off = (size_t)c * 128 + 4 * lane;
        *reinterpret_cast<uint2 *>(qh + off) = make_uint2(wh[0] | (wh[1] << 16), wh[2] | (wh[3] << 16));
        *reinterpret_cast<uint2 *>(ql + off) = make_uint2(wl[0] | (wl[1] << 16), wl[2] | (wl[3] << 16));
        if (res) {
            *reinterpret_cast<uint2 *>(rh + off) = make_uint2(vh[0] | (vh[1] << 16), vh[2] | (vh[3] << 16));
            *reinterpret_cast<uint2 *>(rl + off) = make_uint2(vl[0] | (vl[1] << 16), vl[2] | (vl[3] << 16));
        }
    };
    // pass 2: quantise and store
#pragma unroll
    for (int j = 0; j < KEPT; ++j) {
        const int c = warp + j * WARPS;
        if (c < chunks) quantize_chunk(c, kept[j]);
    }
    for (int c = warp + KEPT * WARPS; c < chunks; c += WARPS) {
        float v[4];
        load(c, v);
        quantize_chunk(c, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
        rsum += __shfl_xor_sync(0xffffffffu, rsum, o);
    }
    if (lane == 0) {
        s_sum[warp] = sum;
        s_rsum[warp] = rsum;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int total = 0, rtotal = 0;
        for (int w = 0; w < WARPS; ++w) {
            total += s_sum[w];
            rtotal += s_rsum[w];
        }
        meta[row] = RowQ{e, total, res ? 1 : 0, rtotal};
    }
    __syncthreads();   // the s_* arrays are reused by the next row
}

// One CTA of WARPS warps per row.  zero (optional): the first CTA also clears zero[0,
// n_zero) (the fused GEMV's queue and expert counters, used by the kernel that follows).
template <typename Src, bool ROTATE, int WARPS>
__global__ void __launch_bounds__(WARPS * 32) quantize_rows_kernel(const Src src, int cols,
                                                                   const int8_t *__restrict__ signs,
                                                                   uint16_t *__restrict__ xq, RowQ *__restrict__ meta,
                                                                   int *__restrict__ zero, int n_zero) {
    chain_entry();
    __shared__ float s_max[WARPS], s_l1[WARPS];
    __shared__ int s_sum[WARPS], s_rsum[WARPS];
    if (zero && blockIdx.x == 0)
        for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero[i] = 0;
    quantize_row<WARPS, Src, ROTATE, 32 / WARPS>(src, blockIdx.x, cols, signs, xq, meta, s_max, s_l1, s_sum, s_rsum);
}

template <bool ROTATE, typename Src, int WARPS = 8>
int launch_quantize_rows(const Src &src, long long rows, int cols, uint16_t *xq, RowQ *meta, cudaStream_t s,
                         int stage, const int8_t *signs = nullptr, int *zero = nullptr, int n_zero = 0) {
    if (rows <= 0) return TQ_OK;
    if (rows > 0x7fffffffll) return TQ_ERR_UNSUPPORTED;
    LaunchScope ls(s, stage);
    launch_chained(quantize_rows_kernel<Src, ROTATE, WARPS>, (unsigned)rows, WARPS * 32, 0, s, src, cols, signs, xq,
                   meta, zero, n_zero);
    return launch_status();
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

// MoE GEMV work item = one CTA of kItemWarps warps: (active expert, 8 strips of 16
// rows, column range, passes of 4 * NB of the expert's routes: NB blocks of 4 routes
// share every decoded weight).  The warps split the item's
// column tiles into contiguous ranges; each streams its range of the 8 strips through
// its own ring, and the warps' integer partial sums are added in shared memory at the
// end of a pass.
//
// GATEUP: item = (active expert, 64 intermediate rows: strips 0..3 of gate, 0..3 of
//         up, column split sp of gu_splits); activations = the tokens' quantised
//         rotated rows (xq, xmeta indexed by token); out = gu [routes][split][2][F]
//         fp32, the split's share of gate x' and up x' (the SwiGLU pass that rotates
//         and quantises h adds the splits in order).  Splits multiply the CTAs of a
//         small batch (gate_up_splits): a 1-token step has 8 active experts, i.e. 128
//         unsplit items for 148 SMs.
// !GATEUP: item = (active expert, 128 output rows); activations = quantised h'
//          (indexed by route); out = y [routes][D] fp32.
constexpr int kNb2MinRoutes = 5;
// routes from which the three GEMV stages run as one fused launch (below: the split form)
constexpr int kFusedMinRoutes = 32;
constexpr int kMaxGateUpSplits = 8;

// Column splits of the gate/up items: enough CTAs for ~3 per SM at the batch's largest
// possible number of active experts (min(E, T k)); 1 from a few tokens on.
inline int gate_up_splits(const tq_moe_layer *L, int T, int k) {
    const long long max_active = min((long long)L->E, (long long)T * k);
    const long long items = max_active * (L->F / 64);
    if (items <= 0) return 1;
    const long long want = (3ll * num_sms() + items - 1) / items;
    return (int)max(1ll, min((long long)kMaxGateUpSplits, min(want, (long long)(L->D / 128))));
}

// Slots of one pass: the routes [tb, next) of the item's expert, one slot per word of
// each route's activation row (a two-word row takes two adjacent slots).
template <int NB>
struct PassSlots {
    int row[4 * NB];      // activation row of the slot (-1: empty, -2: route with an invalid index)
    int word[4 * NB];     // 0: main word, 1: residual word
    int route[4 * NB];    // route offset within the expert (main-word slots)
    int cand[4 * NB];     // candidate routes' rows, then words needed
    int need[4 * NB];
    int next;
};

// Metadata of an activation row (FRESH: written earlier in this launch, plain coherent load).
template <bool FRESH>
__device__ __forceinline__ RowQ load_rowq(const RowQ *p) {
    if constexpr (FRESH) {
        int4 v;
        asm volatile("ld.global.v4.s32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
        return RowQ{v.x, v.y, v.z, v.w};
    } else {
        return *p;
    }
}

// One work item (see above) on the CTA's warp rings.  Returns false if a bounded wait
// gave up (the CTA must stop; every warp drained its copies first).  An expert id the
// layer does not hold raises device flag bit 0 and the item is skipped.  FRESH: activation
// rows and their metadata were written earlier in this launch (x_halves).
template <bool GATEUP, int NB, bool FRESH>
__device__ __forceinline__ bool gemv_item(const tq_moe_layer &L, int item, int splits, const uint16_t *__restrict__ xq,
                                          const RowQ *__restrict__ xmeta, const int32_t *__restrict__ offsets,
                                          const int32_t *__restrict__ perm, const int32_t *__restrict__ active_ids,
                                          int k, int n_routes, float *__restrict__ out, const WarpRing &ring,
                                          uint32_t &parity, ItemRed<NB> &red, PassSlots<NB> &ps) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gq = lane >> 2;
    constexpr int NS = 4 * NB;
    const int per_expert = (GATEUP ? L.F / 64 : L.D / 128) * splits;
    const int a = item / per_expert, sub = (item % per_expert) / splits, sp = item % splits;
    const int e = active_ids[a];
    ExpertRef ex;
    if (!expert_ref(L, e, ex)) {
        if (threadIdx.x == 0) raise_flag(1);
        return true;
    }
    const int cols = GATEUP ? L.D : L.F;
    const int r0 = offsets[e], ne = offsets[e + 1] - r0;
    const int tiles = cols / 16;
    int cb, ce, jb, je;
    split_range(tiles, sp, splits, cb, ce);
    split_range(ce - cb, warp, kItemWarps, jb, je);
    jb += cb;
    je += cb;
    const int cs = lane & 7;
    const uint32_t *strip_lane;
    if (GATEUP)
        strip_lane = (cs < 4 ? ex.gate : ex.up) + (size_t)(sub * 4 + (cs & 3)) * tiles * (8 * ex.K);
    else
        strip_lane = ex.down + (size_t)(sub * 8 + cs) * tiles * (8 * ex.K);

    for (int tb = 0; tb < ne;) {
        // the next NS routes' activation rows and the words each needs
        if (threadIdx.x < NS) {
            const int tt = tb + threadIdx.x;
            int row = -1, need = 0;
            if (tt < ne) {
                if (GATEUP) {
                    const int pr = perm[r0 + tt];
                    row = (pr >= 0 && pr < n_routes) ? pr / k : -2;
                } else {
                    row = r0 + tt;
                }
                need = (row >= 0 && load_rowq<FRESH>(xmeta + row).res) ? 2 : 1;
            }
            ps.cand[threadIdx.x] = row;
            ps.need[threadIdx.x] = need;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            // as many whole routes as fit in the pass's slots (the first always fits)
            int slot = 0, i = 0;
            while (i < NS && ps.need[i] > 0 && slot + ps.need[i] <= NS) {
                for (int w = 0; w < ps.need[i]; ++w, ++slot) {
                    ps.row[slot] = ps.cand[i];
                    ps.word[slot] = w;
                    ps.route[slot] = tb + i;
                }
                ++i;
            }
            for (; slot < NS; ++slot) {
                ps.row[slot] = -1;
                ps.word[slot] = 0;
                ps.route[slot] = -1;
            }
            ps.next = tb + i;
        }
        __syncthreads();
        const uint16_t *xw[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int slot = 4 * b + (gq >> 1);
            const int my_row = ps.row[slot];
            xw[b] = my_row >= 0 ? xq + (size_t)my_row * 4 * cols + (2 * ps.word[slot] + (gq & 1)) * cols : nullptr;
        }
        AccI<NB> acc;
        zero(acc);
        bool ok = stream_any<NB, FRESH>(ex.K, ring, parity, jb, je, strip_lane, xw, acc);
        ok = __syncthreads_and(ok);
        if (!ok) return false;   // every warp drained its copies; the item is left unwritten
        store_partials(acc, red);   // the rings are idle now
        __syncthreads();
        if (GATEUP) {
            for (int i = threadIdx.x; i < 4 * 16 * NS; i += kItemThreads) {
                const int rt = i % NS, row = (i / NS) & 15, st = i / (16 * NS);
                const int xrow = ps.row[rt];
                if (xrow == -1 || ps.word[rt] != 0) continue;
                const int f = (sub * 4 + st) * 16 + row;
                float gv = 0.f, uv = 0.f;    // a route with an invalid index: h = 0
                if (xrow >= 0) {
                    RowQ m = load_rowq<FRESH>(xmeta + xrow);
                    if (sp) m.sum = m.rsum = 0;   // the -255 sum x term is added once, by split 0
                    const int2 g = red_sum(red, st, row, rt), u = red_sum(red, st + 4, row, rt);
                    int2 g2 = make_int2(0, 0), u2 = make_int2(0, 0);
                    if (m.res) {
                        g2 = red_sum(red, st, row, rt + 1);
                        u2 = red_sum(red, st + 4, row, rt + 1);
                    }
                    gv = finish_q(g.x, g.y, m, __half2float(ex.s_gate[f]), g2.x, g2.y);
                    uv = finish_q(u.x, u.y, m, __half2float(ex.s_up[f]), u2.x, u2.y);
                }
                float *o = out + ((size_t)(r0 + ps.route[rt]) * splits + sp) * 2 * L.F + f;
                o[0] = gv;
                o[L.F] = uv;
            }
        } else {
            for (int i = threadIdx.x; i < 8 * 16 * NS; i += kItemThreads) {
                const int rt = i % NS, row = (i / NS) & 15, st = i / (16 * NS);
                const int xrow = ps.row[rt];
                if (xrow < 0 || ps.word[rt] != 0) continue;
                const RowQ m = load_rowq<FRESH>(xmeta + xrow);
                const int2 y = red_sum(red, st, row, rt);
                const int2 y2 = m.res ? red_sum(red, st, row, rt + 1) : make_int2(0, 0);
                const int d = (sub * 8 + st) * 16 + row;
                out[(size_t)xrow * L.D + d] = finish_q(y.x, y.y, m, __half2float(ex.s_down[d]), y2.x, y2.y);
            }
        }
        tb = ps.next;
        __syncthreads();   // the rings and the pass slots are reused by the next pass
    }
    return true;
}

// Waits (thread 0) until *flag is non-zero, polling through L2 with a sleep between
// polls; gives up after kFlagWaitNs (device flag bit 1).  Returns whether it was set.
constexpr uint64_t kFlagWaitNs = 2000000000ull;
// Polls with relaxed loads (an acquire load would invalidate the SM's L1 at every poll,
// under the feet of the other CTAs there); the fence after the load that saw the flag
// makes it an acquire of the producer's release.
__device__ __forceinline__ bool wait_flag(const int *flag) {
    uint64_t t0 = 0;
    for (uint32_t n = 0;; ++n) {
        int v;
        asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v) {
            asm volatile("fence.acq_rel.gpu;" ::: "memory");
            return true;
        }
        if (n == 0) t0 = global_timer_ns();
        else if ((n & 15) == 0 && global_timer_ns() - t0 > kFlagWaitNs) break;
        __nanosleep(200);
    }
    raise_flag(2);
    return false;
}

__device__ __forceinline__ void set_flag(int *flag) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(1) : "memory");
}

// The split form for the smallest batches: one CTA per work item (blockIdx.x; CTAs past
// the active experts' items exit at once), gate/up and down as two launches with the h'
// quantisation between them.  Below kFusedMinRoutes routes a decode step's critical path
// is a chain of dependent global-memory round trips, which kernel boundaries with
// programmatic dependent launch shorten more than the fused kernel's flags do.
template <bool GATEUP, int NB>
__global__ void __launch_bounds__(kItemThreads, NB == 1 ? 5 : 4)
    moe_gemv_items_kernel(const tq_moe_layer L, const uint16_t *__restrict__ xq, const RowQ *__restrict__ xmeta,
                          const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm,
                          const int32_t *__restrict__ active_ids, const int32_t *__restrict__ n_active_p, int k,
                          int n_routes, int gu_splits, float *__restrict__ out) {
    chain_entry();
    extern __shared__ __align__(128) unsigned char smem_raw[];
    ItemSmem &sm_items = *reinterpret_cast<ItemSmem *>(smem_raw);
    ItemRed<NB> &red = *reinterpret_cast<ItemRed<NB> *>(smem_raw);
    __shared__ PassSlots<NB> ps;
    const int warp = threadIdx.x >> 5;
    const int splits = GATEUP ? gu_splits : 1;
    const int per_expert = (GATEUP ? L.F / 64 : L.D / 128) * splits;
    if ((int)blockIdx.x >= *n_active_p * per_expert) return;
    const WarpRing ring{sm_items.buf[warp], sm_items.bar[warp]};
    ring_init(ring);
    uint32_t parity = 0;
    gemv_item<GATEUP, NB, false>(L, blockIdx.x, splits, xq, xmeta, offsets, perm, active_ids, k, n_routes, out, ring,
                                 parity, red, ps);
}

// The routed experts' GEMVs of one decode step in one persistent launch.  Every CTA takes
// work items from a queue (sync[0]): first every gate/up item (expert by expert), then
// every down item.  The CTA that completes the last gate/up item of an expert (counter
// sync[1 + a]) applies the SwiGLU, the rotation and the fixed-point quantisation to that
// expert's routes (h') and raises the expert's ready flag sync[1 + E + a]; a down item
// waits for its expert's flag.  A CTA only waits for work that a running CTA has already
// taken (down items come after every gate/up item in the queue), so the waits end; each is
// bounded all the same.  The items and the quantisation steps are those of the split form
// (moe_gemv_items_kernel, quantize_rows_kernel); only the h' row reductions run over this
// CTA's 4 warps instead of 8.  sync[] is cleared by the x' quantisation kernel before.
template <int NB>
__global__ void __launch_bounds__(kItemThreads, NB == 1 ? 5 : 4)
    moe_gemv_fused_kernel(const tq_moe_layer L, const uint16_t *__restrict__ xq, const RowQ *__restrict__ xmeta,
                          float *__restrict__ gu, uint16_t *__restrict__ hq, RowQ *__restrict__ hmeta,
                          const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm,
                          const int32_t *__restrict__ active_ids, const int32_t *__restrict__ n_active_p, int k,
                          int n_routes, int gu_splits, int *__restrict__ sync, float *__restrict__ y_perm) {
    chain_entry();
    extern __shared__ __align__(128) unsigned char smem_raw[];
    ItemSmem &sm_items = *reinterpret_cast<ItemSmem *>(smem_raw);
    ItemRed<NB> &red = *reinterpret_cast<ItemRed<NB> *>(smem_raw);
    __shared__ PassSlots<NB> ps;
    __shared__ int s_item, s_flag;
    __shared__ float s_max[kItemWarps], s_l1[kItemWarps];
    __shared__ int s_sum[kItemWarps], s_rsum[kItemWarps];
    const int warp = threadIdx.x >> 5;
    const int n_active = *n_active_p;
    const int gu_per = (L.F / 64) * gu_splits, dn_per = L.D / 128;
    const int n_gu = n_active * gu_per, n_all = n_gu + n_active * dn_per;
    const WarpRing ring{sm_items.buf[warp], sm_items.bar[warp]};
    ring_init(ring);
    uint32_t parity = 0;
    for (;;) {
        if (threadIdx.x == 0) s_item = atomicAdd(&sync[0], 1);
        __syncthreads();
        const int item = s_item;
        if (item >= n_all) break;
        if (item < n_gu) {
            if (!gemv_item<true, NB, false>(L, item, gu_splits, xq, xmeta, offsets, perm, active_ids, k, n_routes, gu,
                                            ring, parity, red, ps))
                break;
            // publish this item's g and u; the last of the expert's items turns them into h'
            const int a = item / gu_per;
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) s_flag = atomicAdd(&sync[1 + a], 1) == gu_per - 1;
            __syncthreads();
            if (s_flag) {
                __threadfence();
                const int e = active_ids[a];
                if (e >= 0 && e < L.E) {
                    const int r0 = offsets[e], r1 = offsets[e + 1];
                    // a route's partials (splits x 2 x F fp32) are staged in the idle ring
                    // buffers when they fit, so that their L2 reads overlap.  One pass
                    // computes the final h' values (SwiGLU, signs, rotation) chunk by chunk
                    // into a row buffer -- shared memory after the staged partials when it
                    // fits, else over the route's own split-0 gate partials, whose chunk
                    // has just been read -- and the quantisation reads that buffer twice.
                    const int row_bytes = gu_splits * 2 * L.F * (int)sizeof(float);
                    const int h_bytes = L.F * (int)sizeof(float);
                    const bool staged = row_bytes <= (int)sizeof(sm_items.buf);
                    const bool h_smem = staged && row_bytes + h_bytes <= (int)sizeof(sm_items.buf);
                    unsigned char *st = &sm_items.buf[0][0][0];
                    const int lane = threadIdx.x & 31;
                    for (int r = r0; r < r1; ++r) {
                        float *grow = gu + (size_t)r * gu_splits * 2 * L.F;
                        if (staged) stage_row_async(st, grow, row_bytes);
                        const SwigluFusedSrc src{staged ? reinterpret_cast<const float *>(st) : gu, L.F, gu_splits,
                                                 L.sign_gu, staged};
                        float *hrow = h_smem ? reinterpret_cast<float *>(st + row_bytes) : grow;
                        for (int c = warp; c < L.F / 128; c += kItemWarps) {
                            float v[4];
                            src.load(r, c, lane, v);
                            if (L.sign_h) {   // input side of the two-sided transform: rotate(signs * h)
                                const char4 sg = *reinterpret_cast<const char4 *>(L.sign_h + c * 128 + 4 * lane);
                                v[0] *= sg.x; v[1] *= sg.y; v[2] *= sg.z; v[3] *= sg.w;
                            }
                            fwht128_warp(v, lane);
                            *reinterpret_cast<float4 *>(hrow + (size_t)c * 128 + 4 * lane) = make_float4(v[0], v[1], v[2], v[3]);
                        }
                        __syncthreads();
                        quantize_row<kItemWarps, FinalRowSrc, false, 0>(FinalRowSrc{hrow}, r, L.F, nullptr, hq, hmeta,
                                                                        s_max, s_l1, s_sum, s_rsum);
                    }
                }
                __threadfence();
                __syncthreads();
                if (threadIdx.x == 0) set_flag(&sync[1 + L.E + a]);
            }
        } else {
            const int d = item - n_gu, a = d / dn_per;
            if (threadIdx.x == 0) s_flag = wait_flag(&sync[1 + L.E + a]);
            __syncthreads();
            if (s_flag &&
                !gemv_item<false, NB, true>(L, d, 1, hq, hmeta, offsets, perm, active_ids, k, n_routes, y_perm, ring,
                                            parity, red, ps))
                break;
        }
        __syncthreads();   // s_item and s_flag are rewritten by the next item
    }
}

// ------------------------------------------------------------------------ single GEMV
//
// CTA = (group of 8 strips = 128 rows, column split, pass of 4*NB slots); the 4 warps
// split the CTA's column tiles.  Slots number the words of the batch's rows in order:
// token t's main word is slot t + R(t), R(t) the two-word rows before t, its residual
// word the next slot.  The integer partial sums of all CTAs of a row group are added
// into acc [batch][rows][4] (main H, L, residual H, L) with atomics (exact, so
// order-independent), and gemv_finish_kernel applies the scales.
template <int NB>
__global__ void __launch_bounds__(kItemThreads, 4)
    trellis_gemv_kernel(const uint32_t *__restrict__ bits, int K, int rows, int cols, const uint16_t *__restrict__ xq,
                        const RowQ *__restrict__ meta, int batch, int col_splits, int *__restrict__ acc_out) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    ItemSmem &sm_items = *reinterpret_cast<ItemSmem *>(smem_raw);
    ItemRed<NB> &red = *reinterpret_cast<ItemRed<NB> *>(smem_raw);
    constexpr int NS = 4 * NB;
    __shared__ int s_tok[NS], s_word[NS];
    __shared__ int s_warp[kItemWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gq = lane >> 2;
    // this pass's slots: token ranges per thread, residual-row counts scanned over the CTA
    const int slot0 = blockIdx.z * NS;
    if (threadIdx.x < NS) {
        s_tok[threadIdx.x] = -1;
        s_word[threadIdx.x] = 0;
    }
    const int per = (batch + kItemThreads - 1) / kItemThreads;
    const int t_begin = min(batch, (int)threadIdx.x * per), t_end = min(batch, t_begin + per);
    int mine = 0;
    for (int t = t_begin; t < t_end; ++t) mine += meta[t].res;
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int before = incl - mine;
    for (int w = 0; w < warp; ++w) before += s_warp[w];
    for (int t = t_begin, slot = t_begin + before; t < t_end; ++t) {
        const int words = 1 + meta[t].res;
        for (int w = 0; w < words; ++w, ++slot)
            if (slot >= slot0 && slot < slot0 + NS) {
                s_tok[slot - slot0] = t;
                s_word[slot - slot0] = w;
            }
    }
    __syncthreads();
    if (s_tok[0] < 0) return;   // beyond the batch's last slot (the grid covers two words per row)

    const int n_strips = rows / 16, tiles = cols / 16;
    const WarpRing ring{sm_items.buf[warp], sm_items.bar[warp]};
    ring_init(ring);
    uint32_t parity = 0;
    int cb, ce, jb, je;
    split_range(tiles, blockIdx.y, col_splits, cb, ce);
    split_range(ce - cb, warp, kItemWarps, jb, je);
    jb += cb;
    je += cb;
    const int strip = min((int)blockIdx.x * 8 + (lane & 7), n_strips - 1);   // rows beyond are dropped
    const uint32_t *strip_lane = bits + (size_t)strip * tiles * (8 * K);
    const uint16_t *xw[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const int slot = 4 * b + (gq >> 1);
        const int t = s_tok[slot];
        xw[b] = t >= 0 ? xq + (size_t)t * 4 * cols + (2 * s_word[slot] + (gq & 1)) * cols : nullptr;
    }
    AccI<NB> acc;
    zero(acc);
    bool ok = stream_any<NB>(K, ring, parity, jb, je, strip_lane, xw, acc);
    ok = __syncthreads_and(ok);
    if (!ok) return;
    store_partials(acc, red);
    __syncthreads();
    for (int i = threadIdx.x; i < 8 * 16 * NS; i += kItemThreads) {
        const int rt = i % NS, row = (i / NS) & 15, st = i / (16 * NS);
        const int t = s_tok[rt], r = (blockIdx.x * 8 + st) * 16 + row;
        if (t < 0 || r >= rows) continue;
        const int2 v = red_sum(red, st, row, rt);
        int *dst = acc_out + ((size_t)t * rows + r) * 4 + 2 * s_word[rt];
        atomicAdd(dst, v.x);
        atomicAdd(dst + 1, v.y);
    }
}

__global__ void gemv_finish_kernel(const int *__restrict__ acc, const RowQ *__restrict__ meta,
                                   const __half *__restrict__ scales, int rows, int batch, float *__restrict__ y) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (size_t)rows * batch) return;
    const int t = (int)(i / rows), r = (int)(i % rows);
    const int4 hl = reinterpret_cast<const int4 *>(acc)[i];
    y[i] = finish_q(hl.x, hl.y, meta[t], __half2float(scales[r]), hl.z, hl.w);
}

template <typename Kern>
inline int set_smem(Kern kern, size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) ==
                   cudaSuccess
               ? TQ_OK
               : TQ_ERR_CUDA;
}

inline size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

// Workspace of the single GEMV: quantised rows (4 planes), their RowQ, integer sums.
struct GemvWs {
    uint16_t *xq;
    RowQ *meta;
    int *acc;
};

size_t gemv_ws_bytes(int rows, int cols, int batch) {
    return align256((size_t)batch * 4 * cols * 2) + align256((size_t)batch * sizeof(RowQ)) +
           align256((size_t)rows * batch * 16);
}

GemvWs gemv_ws(void *ws, int rows, int cols, int batch) {
    char *p = reinterpret_cast<char *>(ws);
    GemvWs w;
    w.xq = reinterpret_cast<uint16_t *>(p);
    p += align256((size_t)batch * 4 * cols * 2);
    w.meta = reinterpret_cast<RowQ *>(p);
    p += align256((size_t)batch * sizeof(RowQ));
    w.acc = reinterpret_cast<int *>(p);
    return w;
}

template <int NB>
int run_gemv(const uint32_t *bits, const __half *scales, int K, int rows, int cols, const __half *x, int batch,
             float *y, const GemvWs &w, cudaStream_t s) {
    const size_t smem = sizeof(ItemSmem);
    static PerDeviceFlag configured;
    if (!configured.get()) {
        if (set_smem(trellis_gemv_kernel<NB>, smem)) return TQ_ERR_CUDA;
        configured.set();
    }
    int st = launch_quantize_rows<false>(RowSrc<__half>{x, cols}, batch, cols, w.xq, w.meta, s, kStageGemvQuant);
    if (st) return st;
    if (cudaMemsetAsync(w.acc, 0, (size_t)rows * batch * 16, s) != cudaSuccess) return record_cuda_error("cudaMemsetAsync");
    // the split count is chosen for one word per row; the grid covers up to two words per
    // row, and the CTAs of passes beyond the batch's last slot return at once
    const int groups = (rows / 16 + 7) / 8, passes = (batch + 4 * NB - 1) / (4 * NB), tiles = cols / 16;
    const int want = (4 * num_sms() + groups * passes - 1) / (groups * passes);
    const int splits = max(1, min(want, tiles / (2 * kItemWarps)));
    const int slot_passes = (2 * batch + 4 * NB - 1) / (4 * NB);
    {
        LaunchScope ls(s, kStageGemv);
        trellis_gemv_kernel<NB><<<dim3(groups, splits, slot_passes), kItemThreads, smem, s>>>(
            bits, K, rows, cols, w.xq, w.meta, batch, splits, w.acc);
    }
    st = launch_status();
    if (st) return st;
    const size_t n = (size_t)rows * batch;
    LaunchScope ls(s, kStageGemv);
    gemv_finish_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(w.acc, w.meta, scales, rows, batch, y);
    return launch_status();
}

// ------------------------------------------------------------------------ MoE launch

int validate_layer(const tq_moe_layer *L) {
    if (!L) return TQ_ERR_INVALID_ARG;
    if (L->E < 1 || L->E > 1024 || L->D < 128 || L->F < 128 || L->D % 128 || L->F % 128)
        return TQ_ERR_INVALID_ARG;
    if (L->D > kMaxCols || L->F > kMaxCols) return TQ_ERR_UNSUPPORTED;
    if (L->n_groups < 1 || L->n_groups > 3 || !L->expert_slot) return TQ_ERR_INVALID_ARG;
    if (L->codebook != TQ_CODEBOOK_T16 && L->codebook != TQ_CODEBOOK_PAIR_E4M3) return TQ_ERR_INVALID_ARG;
    const int n_signs = !!L->sign_x + !!L->sign_gu + !!L->sign_h + !!L->sign_y;
    if (n_signs != 0 && n_signs != 4) return TQ_ERR_INVALID_ARG;   // all four or none
    for (const int8_t *sg : {L->sign_x, L->sign_gu, L->sign_h, L->sign_y})
        if (reinterpret_cast<uintptr_t>(sg) & 3) return TQ_ERR_ALIGNMENT;
    for (int g = 0; g < L->n_groups; ++g) {
        const tq_width_group &G = L->groups[g];
        if (G.K < 2 || G.K > 4 || G.n_experts < 0 || G.n_experts > 0xFFFF) return TQ_ERR_INVALID_ARG;
        if (G.n_experts == 0) continue;
        if (!G.gate || !G.up || !G.down || !G.s_gate || !G.s_up || !G.s_down) return TQ_ERR_INVALID_ARG;
        if (!aligned16(G.gate) || !aligned16(G.up) || !aligned16(G.down)) return TQ_ERR_ALIGNMENT;
    }
    return TQ_OK;
}

// Workspace of the MoE GEMV: gate/up partial sums gu [routes][splits][2][F] fp32,
// quantised h' [routes][4][F] half-words (main and residual word planes) and its RowQ
// per route, quantised x' [T][4][D] half-words and its RowQ per token.
struct MoeGemvWs {
    float *gu;
    uint16_t *hq;
    RowQ *hmeta;
    uint16_t *xq;
    RowQ *xmeta;
    int *sync;      // fused kernel: work queue, per-expert gate/up counters and h' flags
};

inline size_t sync_ints(const tq_moe_layer *L) { return 1 + 2 * (size_t)L->E; }

size_t workspace_bytes(const tq_moe_layer *L, int T, int k) {
    const size_t routes = (size_t)T * k;
    return align256(routes * gate_up_splits(L, T, k) * 2 * L->F * 4) + align256(routes * 4 * L->F * 2) +
           align256(routes * sizeof(RowQ)) + align256((size_t)T * 4 * L->D * 2) + align256((size_t)T * sizeof(RowQ)) +
           align256(sync_ints(L) * sizeof(int));
}

MoeGemvWs moe_gemv_ws(const tq_moe_layer *L, int T, int k, void *ws) {
    const size_t routes = (size_t)T * k;
    char *p = reinterpret_cast<char *>(ws);
    MoeGemvWs w;
    w.gu = reinterpret_cast<float *>(p);
    p += align256(routes * gate_up_splits(L, T, k) * 2 * L->F * 4);
    w.hq = reinterpret_cast<uint16_t *>(p);
    p += align256(routes * 4 * L->F * 2);
    w.hmeta = reinterpret_cast<RowQ *>(p);
    p += align256(routes * sizeof(RowQ));
    w.xq = reinterpret_cast<uint16_t *>(p);
    p += align256((size_t)T * 4 * L->D * 2);
    w.xmeta = reinterpret_cast<RowQ *>(p);
    p += align256((size_t)T * sizeof(RowQ));
    w.sync = reinterpret_cast<int *>(p);
    return w;
}

int run_moe_gemv(const tq_moe_layer *L, const __half *x_rot, const int32_t *offsets, const int32_t *perm,
                 const int32_t *active_ids, const int32_t *n_active, int T, int k, float *y_perm,
                 void *ws, cudaStream_t s) {
    const size_t smem = sizeof(ItemSmem);
    static PerDeviceFlag configured;
    static int resident_dev[kMaxDevices][3];   // CTAs per SM of the fused kernel, NB = 1, 2
    int resident_local[3] = {0, 0, 0};
    const int dev = current_device();
    int *resident = dev >= 0 && dev < kMaxDevices ? resident_dev[dev] : resident_local;
    if (!configured.get()) {
        if (set_smem(moe_gemv_fused_kernel<1>, smem) || set_smem(moe_gemv_fused_kernel<2>, smem) ||
            set_smem(moe_gemv_items_kernel<true, 1>, smem) || set_smem(moe_gemv_items_kernel<false, 1>, smem) ||
            set_smem(moe_gemv_items_kernel<true, 2>, smem) || set_smem(moe_gemv_items_kernel<false, 2>, smem))
            return TQ_ERR_CUDA;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident[1], moe_gemv_fused_kernel<1>, kItemThreads,
                                                          smem) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident[2], moe_gemv_fused_kernel<2>, kItemThreads,
                                                          smem) != cudaSuccess)
            return record_cuda_error("cudaOccupancyMaxActiveBlocksPerMultiprocessor");
        configured.set();
    }
    const int routes = T * k;
    const MoeGemvWs w = moe_gemv_ws(L, T, k, ws);
    const long long max_active = min(L->E, routes);
    const int splits = gate_up_splits(L, T, k);
    const long long max_items = max_active * ((long long)(L->F / 64) * splits + L->D / 128);
    // 8 routes per pass once a batch averages kNb2MinRoutes or more routes per expert
    // (each decoded weight then feeds twice the MMAs instead of being decoded twice)
    const bool nb2 = routes >= kNb2MinRoutes * min(L->E, routes);
    const int nb = nb2 ? 2 : 1;
    if (routes < kFusedMinRoutes) {
        // split form: x' quantisation, gate/up items, h' quantisation, down items
        const unsigned gu_items = (unsigned)(max_active * (L->F / 64) * splits);
        const unsigned dn_items = (unsigned)(max_active * (L->D / 128));
        int st = launch_quantize_rows<false>(RowSrc<__half>{x_rot, L->D}, T, L->D, w.xq, w.xmeta, s, kStageGemvQuant);
        if (st) return st;
        {
            LaunchScope ls(s, kStageMoeGemv);
            if (nb2)
                launch_chained(moe_gemv_items_kernel<true, 2>, gu_items, kItemThreads, smem, s, *L, w.xq, w.xmeta,
                               offsets, perm, active_ids, n_active, k, routes, splits, w.gu);
            else
                launch_chained(moe_gemv_items_kernel<true, 1>, gu_items, kItemThreads, smem, s, *L, w.xq, w.xmeta,
                               offsets, perm, active_ids, n_active, k, routes, splits, w.gu);
        }
        st = launch_status();
        if (st) return st;
        st = launch_quantize_rows<true>(SwigluSrc{w.gu, L->F, splits, L->sign_gu}, routes, L->F, w.hq, w.hmeta, s,
                                        kStageRotateH, L->sign_h);
        if (st) return st;
        LaunchScope ls(s, kStageGemvDown);
        if (nb2)
            launch_chained(moe_gemv_items_kernel<false, 2>, dn_items, kItemThreads, smem, s, *L, w.hq, w.hmeta, offsets,
                           perm, active_ids, n_active, k, routes, 1, y_perm);
        else
            launch_chained(moe_gemv_items_kernel<false, 1>, dn_items, kItemThreads, smem, s, *L, w.hq, w.hmeta, offsets,
                           perm, active_ids, n_active, k, routes, 1, y_perm);
        return launch_status();
    }
    // x' rows to fixed point; the same launch clears the fused kernel's queue and counters
    int st = launch_quantize_rows<false>(RowSrc<__half>{x_rot, L->D}, T, L->D, w.xq, w.xmeta, s, kStageGemvQuant,
                                         nullptr, w.sync, (int)sync_ints(L));
    if (st) return st;
    const long long slots = (long long)max(1, resident[nb]) * num_sms();
    const unsigned grid = (unsigned)max(1ll, min(slots, max_items));
    LaunchScope ls(s, kStageMoeGemv);
    if (nb2)
        launch_chained(moe_gemv_fused_kernel<2>, grid, kItemThreads, smem, s, *L, w.xq, w.xmeta, w.gu, w.hq, w.hmeta,
                       offsets, perm, active_ids, n_active, k, routes, splits, w.sync, y_perm);
    else
        launch_chained(moe_gemv_fused_kernel<1>, grid, kItemThreads, smem, s, *L, w.xq, w.xmeta, w.gu, w.hq, w.hmeta,
                       offsets, perm, active_ids, n_active, k, routes, splits, w.sync, y_perm);
    return launch_status();
}

}  // namespace tq

using namespace tq;

TQ_API size_t trellis_gemv_workspace_size(int rows, int cols, int batch) {
    if (rows < 0 || cols < 0 || batch < 0 || rows % 16 || cols % 128 || cols > kMaxCols) return 0;
    return gemv_ws_bytes(rows, cols, batch);
}

TQ_API int trellis_gemv(const uint32_t *bits, const uint16_t *scales, int K, int rows, int cols,
                        const uint16_t *x_rot, int batch, float *y, void *ws, size_t ws_bytes, tq_stream stream) {
    if (K < 2 || K > 4 || rows < 0 || cols < 0 || rows % 16 || cols % 128 || batch < 0)
        return TQ_ERR_INVALID_ARG;
    if (cols > kMaxCols || batch > 65535) return TQ_ERR_UNSUPPORTED;
    if (rows == 0 || batch == 0) return TQ_OK;
    if (cols == 0) return TQ_ERR_INVALID_ARG;
    if (!bits || !scales || !x_rot || !y) return TQ_ERR_INVALID_ARG;
    if (!aligned16(bits) || !aligned16(x_rot)) return TQ_ERR_ALIGNMENT;
    if (!ws || ws_bytes < gemv_ws_bytes(rows, cols, batch)) return TQ_ERR_WORKSPACE;
    if (!aligned16(ws)) return TQ_ERR_ALIGNMENT;
    cudaStream_t s = (cudaStream_t)stream;
    const __half *sc = reinterpret_cast<const __half *>(scales);
    const __half *x = reinterpret_cast<const __half *>(x_rot);
    const GemvWs w = gemv_ws(ws, rows, cols, batch);
    if (batch <= 4) return run_gemv<1>(bits, sc, K, rows, cols, x, batch, y, w, s);
    return run_gemv<2>(bits, sc, K, rows, cols, x, batch, y, w, s);
}

namespace tq {
size_t gemm_workspace_bytes(const tq_moe_layer *L, int T, int k);
}

TQ_API size_t moe_trellis_workspace_size(const tq_moe_layer *layer, int T, int k) {
    if (validate_layer(layer) != TQ_OK || T < 0 || k < 1) return 0;
    const size_t gemv = workspace_bytes(layer, T, k), gemm = tq::gemm_workspace_bytes(layer, T, k);
    return gemv > gemm ? gemv : gemm;
}

// Every argument of a MoE call except the workspace.
int moe_validate_args(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                      const int32_t *perm, const int32_t *active_ids, const int32_t *n_active, int T,
                      int k, float *y_perm) {
    int st = validate_layer(layer);
    if (st) return st;
    if (T < 0 || k < 1 || k > layer->E) return TQ_ERR_INVALID_ARG;
    if ((long long)T * k > (1ll << 30)) return TQ_ERR_UNSUPPORTED;
    if (T == 0) return TQ_OK;
    if (!x_rot || !offsets || !perm || !active_ids || !n_active || !y_perm) return TQ_ERR_INVALID_ARG;
    if (!aligned16(x_rot) || !aligned16(y_perm)) return TQ_ERR_ALIGNMENT;
    return TQ_OK;
}

int moe_validate_call(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                      const int32_t *perm, const int32_t *active_ids, const int32_t *n_active, int T,
                      int k, float *y_perm, void *ws, size_t ws_bytes) {
    int st = moe_validate_args(layer, x_rot, offsets, perm, active_ids, n_active, T, k, y_perm);
    if (st || T == 0) return st;
    if (!ws || ws_bytes < workspace_bytes(layer, T, k)) return TQ_ERR_WORKSPACE;
    if (!aligned16(ws)) return TQ_ERR_ALIGNMENT;
    return TQ_OK;
}

TQ_API int moe_trellis_gemv(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                            const int32_t *perm, const int32_t *active_ids, const int32_t *n_active, int T,
                            int k, float *y_perm, void *ws, size_t ws_bytes, tq_stream stream) {
    int st = moe_validate_call(layer, x_rot, offsets, perm, active_ids, n_active, T, k, y_perm, ws, ws_bytes);
    if (st || T == 0) return st;
    if (layer->codebook != TQ_CODEBOOK_T16) return TQ_ERR_UNSUPPORTED;   // the GEMV decodes T16 only
    const __half *x = reinterpret_cast<const __half *>(x_rot);
    cudaStream_t s = (cudaStream_t)stream;
    return run_moe_gemv(layer, x, offsets, perm, active_ids, n_active, T, k, y_perm, ws, s);
}
