// Prefill-sized routed-expert GEMM on the 5th-generation tensor cores (tcgen05).
//
// Same computation as moe_trellis_gemv (T16 codebook and 16x16 column-major tiles,
// "How T16 works" items 1, 2 and 4 of the dsx T16 card; SwiGLU experts with fused
// gate/up post-processing, its "October 25 runtime checkpoint"), for hundreds to
// thousands of routes per expert, where each decoded weight feeds a 256-route MMA.
//
// Data flow of one launch (gate/up or down):
//   * The routes' activations are a route-ordered fp16 matrix B_all [T*k][Kdim]
//     (gate/up: the rotated tokens gathered to their route rows by route_rows_kernel;
//     down: the rotated h'), with per-route row sums.
//   * A CTA owns one tile: (expert, block of <= 256 of its routes, 128 weight rows).
//     Per K-block of 64 columns (4 stages in flight):
//       - producer warp: bulk-copies the 8 strips' 4 trellis tiles (the bit stream)
//         and TMA-loads the routes' 64-column slab (128-byte swizzle) into the stage;
//       - two decode groups of 4 warps (alternating K-blocks) decode the 8192 weights
//         of the stage into the K-major 128-byte-swizzled A buffer as fp16 subnormals
//         t * 2^-24 (exact; t = lo + hi of the T16 product);
//       - one thread issues 4 tcgen05.mma (M=128, N<=256, K=16, fp32 accumulator in
//         tensor memory) and commits them to the stage's "empty" barrier.
//   * Epilogue (4 warps, one per tensor-memory lane quarter): tcgen05.ld of the
//     accumulator, D -> s * 2^-12 * (2^24 D - 255 * rowsum), times the route row's
//     power-of-two scale for the down projection (h' rows are stored as fp16 h' / 2^e,
//     largest magnitude in [2^14, 2^15), so any finite fp32 h keeps fp16's relative
//     precision and never overflows), then
//       gate/up: strips are interleaved gate/up per 16 rows, so lane l and l^16 hold g
//                and u of the same intermediate row: h = silu(g) * u (fp32);
//       down:    y_perm (fp32).
// Every wait on an mbarrier is bounded; a wait that gives up raises device flag bit 1,
// the CTA stops issuing work, drains what it issued and releases its tensor memory.
#include "tq_common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

namespace tq {

constexpr int kGBM = 128;          // weight rows per MMA tile (one accumulator)
constexpr int kGTiles = 2;         // weight tiles per CTA: both share every activation slab
constexpr int kGBN = 256;          // max routes per CTA
constexpr int kGRowBytes = 128;    // bytes of one operand row per K-block (128-byte swizzle)
constexpr int kGGroups = 2;        // K-block slots: K-block kb is decoded into A slot kb % 2
constexpr int kGDecodeGroups = 2 * kGGroups;   // 4-warp groups: (K-block parity, weight tile)
constexpr int kGBitsBytes = 48 * 1024;   // bit-stream ring: 6 stages (T16) or 3 (pair trellis)
constexpr int kGBStages = 3;       // activation (B) ring
constexpr int kGKbRing = 4;        // K-block barrier ring: > the A and B reuse distances
constexpr int kGDecodeWarps = 4 * kGDecodeGroups;
constexpr int kGFirstDecodeWarp = 3;   // warp 0: bit-stream producer, 1: MMA, 2: B producer
constexpr int kGThreads = (kGFirstDecodeWarp + kGDecodeWarps) * 32;
constexpr int kGStrips = 8 * kGTiles;  // 16-row strips per CTA
constexpr int kGBoxes = 4;         // TMA boxes of 32, 64, 128, 256 rows
constexpr uint32_t kGTmemCols = 512;   // two 256-column fp32 accumulators
constexpr int kGMaxBitsStages = 6;

// Per-codebook shape of a K-block.  T16 weights become fp16 operands (64 columns per
// 128-byte row, kind::f16 MMAs of K = 16); pair-trellis weights become E4M3 operands (128
// columns per row, kind::f8f6f4 MMAs of K = 32).  Either way a K-block is 4 MMAs per
// weight tile and the operand rows are 128 bytes, so the shared-memory layout, the
// swizzle and the descriptors are the same.
template <bool FP8>
struct GemmShape {
    static constexpr int kTiles = FP8 ? 8 : 4;               // 16-column tiles per K-block
    static constexpr int kCols = 16 * kTiles;                // K columns per K-block
    static constexpr int kSlot = kTiles * 128;               // bit-stream bytes per strip (K <= 4)
    static constexpr int kStage = kGStrips * kSlot;
    static constexpr int kBitsStages = kGBitsBytes / kStage; // 6 or 3
    static_assert(kBitsStages >= 2 && kBitsStages <= kGMaxBitsStages, "bit-stream ring");
};

struct __align__(1024) GemmSmem {
    unsigned char a[kGGroups][kGTiles][kGBM * kGRowBytes];  // 2 x 16 KB per decode group, 1024-aligned
    unsigned char b[kGBStages][kGBN * kGRowBytes];          // 32 KB per stage
    unsigned char bits[kGBitsBytes];                        // bit-stream stages (GemmShape)
    uint64_t bits_full[kGMaxBitsStages];       // producer -> decoders (count 1 + bytes)
    uint64_t bits_empty[kGMaxBitsStages];      // decoders -> producer (count 8)
    // One barrier pair per K-block (ring of kGKbRing): kb_ready completes when the 8
    // decode warps of the K-block have arrived and its activation slab has landed (the
    // MMA thread waits once per K-block); kb_done is the MMA commit, waited by the
    // decoders before reusing the A slot (K-block kb + 2) and by the activation
    // producer before reusing the slab stage (kb + 3).
    uint64_t kb_ready[kGKbRing];
    uint64_t kb_done[kGKbRing];
    uint64_t acc_full;                         // MMA -> epilogue
    uint64_t mma_done;                         // MMA drain on early exit
    float2 rs[kGDecodeWarps][kGBN / 2];        // epilogue: each decode warp's route (row sum, scale)
    uint32_t tmem_base;
    int32_t abort;                             // a role gave up
};

// dynamic shared memory of one CTA (plus 1 KB for the 1024-byte alignment) must fit the
// 227 KB a CTA may use on sm_100
static_assert(sizeof(GemmSmem) + 1024 <= 227 * 1024, "GEMM shared memory exceeds the per-CTA limit");

struct GemmMaps {
    CUtensorMap b[kGBoxes];               // route-ordered activations, box rows 32..256
    // bit streams of each width group as [expert][strip][words] (uint32), box
    // {4 tiles, 8 or 16 strips, 1}: gate/up launch: first = gate, second = up (8
    // strips each); down launch: first = down (16 strips).
    CUtensorMap bits_first[3];
    CUtensorMap bits_second[3];
};

// ------------------------------------------------------------------------------ PTX

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols) : "memory");
}

// K-major operand in shared memory with the 128-byte swizzle: rows of 128 B, 8-row
// atoms 1024 B apart (SBO), start address advanced by 32 B per K=16 step.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;                 // leading byte offset (unused for this layout)
    d |= (uint64_t)(1024u >> 4) << 32;       // stride byte offset: 8-row atoms
    d |= (uint64_t)1u << 46;                 // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                 // SWIZZLE_128B
    return d;
}

// kind::f16 instruction descriptor: fp16 A and B (K-major), fp32 D, M = 128, N.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kGBM >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// E4M3 x E4M3 -> fp32 (kind::f8f6f4, K = 32); the instruction descriptor's A and B format
// fields are 0 (E4M3) in the same bit positions as kind::f16's fp16.
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns; thread i of the warp gets lane base+i.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------------------ decode

__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Product of the window at compile-time bit offset O, bytes [0, 0, lo, hi].
template <int O, int NS>
__device__ __forceinline__ uint32_t prod_hi(const uint32_t (&v)[NS]) {
    constexpr int wi = O >> 5, sh = O & 31;
    uint32_t bottom;
    if constexpr (sh == 0) bottom = v[wi];
    else bottom = funnel_r(v[wi], v[wi + 1], sh);
    return bottom * (kT16Mult << 16);
}

// Rows R of the lane's 4 columns -> 4 fp16 subnormals t * 2^-24, stored (8 bytes) into
// the swizzled A stage: row m = row0 + R (row0 a multiple of 16), so the swizzle
// depends on R only and addr[R & 7] + (R >> 3) * 1024 is the store address.
template <int K, int R>
__device__ __forceinline__ void decode_rows(const uint32_t (&v)[2 * K + 1], const uint32_t (&addr)[8]) {
    if constexpr (R < 16) {
        const uint32_t p0 = prod_hi<0 * 16 * K + K * R>(v), p1 = prod_hi<1 * 16 * K + K * R>(v);
        const uint32_t p2 = prod_hi<2 * 16 * K + K * R>(v), p3 = prod_hi<3 * 16 * K + K * R>(v);
        const uint32_t ab = hadd2_u32(prmt(p0, p1, 0x4602u), prmt(p0, p1, 0x5713u));
        const uint32_t cd = hadd2_u32(prmt(p2, p3, 0x4602u), prmt(p2, p3, 0x5713u));
        asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr[R & 7] + (R >> 3) * 1024), "r"(ab), "r"(cd)
                     : "memory");
        decode_rows<K, R + 1>(v, addr);
    }
}

// Decode one (strip slot, column tile, lane quarter) cell of a K-block: 16 rows x 4
// columns into the swizzled A stage of its weight tile.
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

template <int K>
__device__ __forceinline__ void decode_cell(uint32_t bits_stage_s, uint32_t a_tile_s, int sig_in_tile, int row,
                                            int j, int t4) {
    constexpr int TB = 32 * K;
    const uint32_t tile = bits_stage_s + row * (4 * TB) + j * TB;   // rows packed by the tensor copy
    uint32_t v[2 * K + 1];
    if constexpr (K == 2) {
        uint4 a = lds128(tile + 16 * t4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else if constexpr (K == 3) {
        const uint32_t q = tile + 24 * t4;
        uint2 a = lds64(q), b = lds64(q + 8), c = lds64(q + 16);
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y; v[4] = c.x; v[5] = c.y;
    } else {
        const uint32_t q = tile + 32 * t4;
        uint4 a = lds128(q), b = lds128(q + 16);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    v[2 * K] = lds32(tile + 8 * K * ((t4 + 1) & 3));
    const int kc = 16 * j + 4 * t4;   // first K column of the lane within the K-block
    const int chunk = kc >> 3, half_off = (kc & 7) * 2;
    uint32_t addr[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) addr[r] = a_tile_s + (16 * sig_in_tile + r) * 128 + ((chunk ^ r) << 4) + half_off;
    decode_rows<K, 0>(v, addr);
}

// Pair-trellis (E4M3) cell: 16 rows x 4 columns (quarter t4 of column tile j of strip
// slot sig) decoded to E4M3 bytes and stored, 4 bytes per row, into the K-major
// 128-byte-swizzled A buffer: row m = 16 sig + r, K byte 16 j + 4 t4 (16-byte chunk j,
// swizzled by m mod 8).  Stage rows are 8 column tiles of one strip.
template <int K>
__device__ __forceinline__ void decode_cell_e4m3(uint32_t bits_stage_s, uint32_t a_tile_s, int sig, int row, int j,
                                                 int t4) {
    constexpr int TB = 32 * K;
    const uint32_t tile = bits_stage_s + row * (8 * TB) + j * TB;
    uint32_t v[2 * K + 1];
    if constexpr (K == 2) {
        uint4 a = lds128(tile + 16 * t4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else if constexpr (K == 3) {
        const uint32_t q = tile + 24 * t4;
        uint2 a = lds64(q), b = lds64(q + 8), c = lds64(q + 16);
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y; v[4] = c.x; v[5] = c.y;
    } else {
        const uint32_t q = tile + 32 * t4;
        uint4 a = lds128(q), b = lds128(q + 16);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    v[2 * K] = lds32(tile + 8 * K * ((t4 + 1) & 3));
    uint32_t rows[16];
    pair_cell_rows<K, 0>(v, rows);
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const uint32_t addr = a_tile_s + (16 * sig + r) * 128 + ((j ^ (r & 7)) << 4) + 4 * t4;
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(rows[r]) : "memory");
    }
}

// Decode weight tile t of one K-block (8 strips x 8 column tiles) of the pair trellis: the
// 4-warp group's 128 threads take 2 cells each (same quarter t4, column tiles j, j + 4).
template <int K, bool GATEUP>
__device__ __forceinline__ void decode_tile_e4m3(uint32_t bits_stage_s, uint32_t a_tile_s, int t, int wl, int lane) {
    const int t4 = lane & 3;
    const int base = wl * 8 + (lane >> 2);   // 0..31: (strip slot, column tile mod 4)
    const int sig = base >> 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int j = (base & 3) + 4 * h;
        const int row = GATEUP ? (sig & 1) * 8 + 4 * t + (sig >> 1) : 8 * t + sig;
        decode_cell_e4m3<K>(bits_stage_s, a_tile_s, sig, row, j, t4);
    }
}

// Decode weight tile t of one K-block (8 strips x 4 column tiles) with a 4-warp group:
// thread (wl, lane) takes one (strip slot, column tile, quarter) cell.  Rows of the
// bit-stream stage: gate/up: [8 gate strips][8 up strips] of the tile pair (tile t,
// slot sl -> row (sl & 1) * 8 + 4t + (sl >> 1)); down: 16 consecutive strips.
template <int K, bool GATEUP>
__device__ __forceinline__ void decode_tile(uint32_t bits_stage_s, uint32_t a_tile_s, int t, int wl, int lane) {
    const int cell = wl * 8 + (lane >> 2);   // 0..31: (strip slot, column tile)
    const int sig = cell >> 2, j = cell & 3, t4 = lane & 3;
    const int row = GATEUP ? (sig & 1) * 8 + 4 * t + (sig >> 1) : 8 * t + sig;
    decode_cell<K>(bits_stage_s, a_tile_s, sig, row, j, t4);
}

// ------------------------------------------------------------------------------ kernel

struct GemmArgs {
    tq_moe_layer L;
    const int32_t *offsets;
    const int32_t *tiles;        // [0] = count, then (expert, first route) pairs
    const float *rowsum;         // [T*k] sum of each route's activation row
    const float *rowscale;       // [T*k] power-of-two scale of each route's row, or null (1)
    float *out;                  // gate/up: h [T*k][F] (raw_gu: g, u [T*k][2][F]); down: y [T*k][D]
    int kdim;                    // D (gate/up) or F (down)
    int raw_gu;                  // gate/up of the two-sided transform: store g and u, not h
};

template <bool GATEUP, bool FP8>
__global__ void __launch_bounds__(kGThreads, 1)
    moe_gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmArgs args) {
    using SH = GemmShape<FP8>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    // The stage buffers need 1024-byte alignment (128-byte swizzle atoms).  Offset the
    // __shared__ array itself (no round trip through an integer) so that the compiler
    // keeps shared-memory instructions for every access derived from it.
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    GemmSmem &sm = *reinterpret_cast<GemmSmem *>(smem_raw + pad);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const tq_moe_layer &L = args.L;

    const int t = blockIdx.y, mt = blockIdx.x;
    if (t >= args.tiles[0]) return;
    const int e = args.tiles[1 + 2 * t], n0 = args.tiles[2 + 2 * t];
    ExpertRef ex;
    if (!expert_ref(L, e, ex)) {
        if (threadIdx.x == 0) raise_flag(1);
        return;
    }
    const int r0 = args.offsets[e], ne = args.offsets[e + 1] - r0;
    const int n = min(kGBN, ne - n0);
    if (n <= 0) return;
    int box = 0;
    while ((32 << box) < n) ++box;          // box rows 32 << box >= n
    const int nmma = max(16, (n + 15) & ~15);
    const int num_kb = args.kdim / SH::kCols;

    if (threadIdx.x == 0) {
        for (int i = 0; i < SH::kBitsStages; ++i) {
            mbar_init(&sm.bits_full[i], 1);
            mbar_init(&sm.bits_empty[i], 8);
        }
        for (int i = 0; i < kGKbRing; ++i) {
            mbar_init(&sm.kb_ready[i], 8 + 1);   // 8 decode warps + the producer's expect_tx
            mbar_init(&sm.kb_done[i], 1);
        }
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.mma_done, 1);
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, kGTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = sm.tmem_base;
    // a wait that gave up anywhere stops every role: check the shared flag too
    auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
        const bool ok = __all_sync(0xffffffffu, mbar_wait_sleep(bar, parity));
        if (!ok) sm.abort = 1;
        // one answer for the whole warp, so that its lanes leave their loops together
        return ok && !__any_sync(0xffffffffu, *(volatile int32_t *)&sm.abort != 0);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ bit-stream producer
        const int K = ex.K;
        const int row_bytes = SH::kTiles * 32 * K;            // the K-block's column tiles of one strip
        const CUtensorMap *m1 = &maps.bits_first[ex.group], *m2 = &maps.bits_second[ex.group];
        const int strip0 = GATEUP ? mt * 8 : mt * 16;         // first strip of the CTA
        int issued = 0;
        for (int kb = 0; kb < num_kb; ++kb) {
            const int i = kb % SH::kBitsStages;
            if (kb >= SH::kBitsStages && !wait(&sm.bits_empty[i], ((kb / SH::kBitsStages) - 1) & 1)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&sm.bits_full[i], (uint32_t)kGStrips * row_bytes);
                const int x = kb * SH::kTiles * 8 * K;        // word offset of the K-block
                unsigned char *stage = sm.bits + i * SH::kStage;
                if (GATEUP) {
                    tma_load_3d(stage, m1, x, strip0, ex.index, &sm.bits_full[i]);
                    tma_load_3d(stage + 8 * row_bytes, m2, x, strip0, ex.index, &sm.bits_full[i]);
                } else {
                    tma_load_3d(stage, m1, x, strip0, ex.index, &sm.bits_full[i]);
                }
            }
            __syncwarp();
            ++issued;
        }
        // drain: every issued copy has landed before the CTA can exit
        for (int kb = max(0, issued - SH::kBitsStages); kb < issued; ++kb)
            mbar_wait_sleep(&sm.bits_full[kb % SH::kBitsStages], (kb / SH::kBitsStages) & 1);
    } else if (warp == 2) {
        // ------------------------------------------------------------ activation producer
        int issued = 0;
        for (int kb = 0; kb < num_kb; ++kb) {
            const int i = kb % kGBStages;
            const int pk = kb - kGBStages;    // the K-block that last used stage i
            if (pk >= 0 && !wait(&sm.kb_done[pk % kGKbRing], (pk / kGKbRing) & 1)) break;
            uint64_t *ready = &sm.kb_ready[kb % kGKbRing];
            if (lane == 0) {
                mbar_arrive_expect_tx(ready, (32u << box) * 128u);
                tma_load_2d(sm.b[i], &maps.b[box], kb * SH::kCols, r0 + n0, ready);
            }
            __syncwarp();
            ++issued;
        }
        // drain: the copies land within microseconds (these barriers also count the
        // decoders, so after an abort they may only complete by the wait's limit)
        for (int kb = max(0, issued - kGBStages); kb < issued; ++kb)
            mbar_wait_sleep(&sm.kb_ready[kb % kGKbRing], (kb / kGKbRing) & 1);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // One lane runs the loop: one bounded wait per K-block, 2 x 4 MMAs whose
        // descriptors step by 32 B (2 in 16-byte units) from per-slot bases, one commit.
        const uint32_t idesc = umma_idesc_f16(nmma);
        bool ok = true;
        if (lane == 0) {
            // the start-address field holds address >> 4 (14 bits, shared memory < 256 KB)
            const uint64_t a_desc0 = umma_desc_sw128(smem_u32(sm.a[0][0]));
            const uint64_t b_desc0 = umma_desc_sw128(smem_u32(sm.b[0]));
            constexpr uint32_t a_step = sizeof(sm.a[0][0]) >> 4, b_step = sizeof(sm.b[0]) >> 4;
            for (int kb = 0; kb < num_kb; ++kb) {
                const int g = kb % kGGroups, i = kb % kGBStages;
                if (!mbar_wait_sleep(&sm.kb_ready[kb % kGKbRing], (kb / kGKbRing) & 1) ||
                    *(volatile int32_t *)&sm.abort) {
                    sm.abort = 1;
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int t = 0; t < kGTiles; ++t)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {   // 32-byte K steps: K = 16 fp16 or 32 E4M3
                        const uint64_t ad = a_desc0 + (uint64_t)((g * kGTiles + t) * a_step + 2 * k);
                        const uint64_t bd = b_desc0 + (uint64_t)(i * b_step + 2 * k);
                        if constexpr (FP8) umma_e4m3(tmem_d + t * kGBN, ad, bd, idesc, (kb | k) != 0);
                        else umma_f16(tmem_d + t * kGBN, ad, bd, idesc, (kb | k) != 0);
                    }
                umma_commit(&sm.kb_done[kb % kGKbRing]);
            }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (lane == 0) umma_commit(ok ? &sm.acc_full : &sm.mma_done);
        __syncwarp();
        if (!ok) mbar_wait_sleep(&sm.mma_done, 0);
    } else {
        // ------------------------------------------------------------ decoders
        // group dg: K-blocks of parity dg >> 1 (A slot), weight tile dg & 1
        const int dw = warp - kGFirstDecodeWarp;
        const int dg = dw >> 2, wl = dw & 3;
        const int slot = dg >> 1, tile = dg & 1;
        const uint32_t a_s = smem_u32(sm.a[slot][tile]);
        for (int kb = slot; kb < num_kb; kb += kGGroups) {
            const int i = kb % SH::kBitsStages;
            if (!wait(&sm.bits_full[i], (kb / SH::kBitsStages) & 1)) break;
            const int pk = kb - kGGroups;     // the K-block that last used this A slot
            if (pk >= 0 && !wait(&sm.kb_done[pk % kGKbRing], (pk / kGKbRing) & 1)) break;
            const uint32_t bits_s = smem_u32(sm.bits + i * SH::kStage);
            if constexpr (FP8) {
                if (ex.K == 2) decode_tile_e4m3<2, GATEUP>(bits_s, a_s, tile, wl, lane);
                else if (ex.K == 3) decode_tile_e4m3<3, GATEUP>(bits_s, a_s, tile, wl, lane);
                else decode_tile_e4m3<4, GATEUP>(bits_s, a_s, tile, wl, lane);
            } else {
                if (ex.K == 2) decode_tile<2, GATEUP>(bits_s, a_s, tile, wl, lane);
                else if (ex.K == 3) decode_tile<3, GATEUP>(bits_s, a_s, tile, wl, lane);
                else decode_tile<4, GATEUP>(bits_s, a_s, tile, wl, lane);
            }
            fence_proxy_async();      // make the generic-proxy writes visible to the MMA
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.kb_ready[kb % kGKbRing]);
                mbar_arrive(&sm.bits_empty[i]);
            }
        }
        // ------------------------------------------------------------ epilogue
        // group dg reads half (dg >> 1) of the columns of weight tile dg & 1, one warp
        // per tensor-memory lane quarter.  The warp's route row sums (into its own
        // shared-memory row) and its rows' scales are loaded before the accumulator
        // wait, so that no global load sits in the store loop.
        {
            const int tt = tile;
            const int q = warp & 3;
            const int row = 32 * q + lane;  // weight row of tile tt = tensor-memory lane
            const int mtile = mt * kGTiles + tt;
            const int half_cols = ((nmma / 16 + 1) / 2) * 16;
            const int cb = slot * half_cols, ce = min(nmma, cb + half_cols);
            float2 *rsw = sm.rs[warp - kGFirstDecodeWarp];
            for (int i = lane; i < ce - cb; i += 32) {
                const int col = cb + i;
                float2 v = make_float2(0.f, 1.f);
                if (col < n) {
                    if (args.rowsum) v.x = args.rowsum[r0 + n0 + col];
                    if (args.rowscale) v.y = args.rowscale[r0 + n0 + col];
                }
                rsw[i] = v;
            }
            const int f = (mtile * 4 + q) * 16 + (lane & 15);
            const int hi = lane >> 4;
            const float kappa = FP8 ? kKappa8 : kKappa;
            float sk0, sk1 = 0.f;            // the lane's row scales times the codebook's normaliser
            if (GATEUP) {
                sk0 = __half2float(ex.s_gate[f]) * kappa;
                sk1 = __half2float(ex.s_up[f]) * kappa;
            } else {
                sk0 = __half2float(ex.s_down[mtile * kGBM + row]) * kappa;
            }
            __syncwarp();
            if (wait(&sm.acc_full, 0)) {
                tc_fence_after();
                const uint32_t taddr = tmem_d + ((uint32_t)(32 * q) << 16) + (uint32_t)(tt * kGBN);
                for (int c0 = cb; c0 < ce; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld16(taddr + c0, v);
                    const float2 *rsc = rsw + (c0 - cb);
                    if (GATEUP) {
                        // lane l < 16 holds the gate row of output f, lane l + 16 the up row;
                        // one exchange per column pair gives lane l both values of column c
                        // and lane l + 16 both values of column c + 1
#pragma unroll
                        for (int c = 0; c < 16; c += 2) {
                            const float mine0 = __uint_as_float(v[c]), mine1 = __uint_as_float(v[c + 1]);
                            const float other = __shfl_xor_sync(0xffffffffu, hi ? mine0 : mine1, 16);
                            const float graw = hi ? other : mine0, uraw = hi ? mine1 : other;
                            const int col = c0 + c + hi;
                            if (col < n) {
                                const int route = r0 + n0 + col;
                                float g, u;
                                if constexpr (FP8) {
                                    // E4M3 codes are signed values; the route row's scale
                                    const float xs = rsc[c + hi].y;
                                    g = (sk0 * xs) * graw;
                                    u = (sk1 * xs) * uraw;
                                } else {
                                    const float sx = rsc[c + hi].x;
                                    g = sk0 * fmaf(16777216.0f, graw, -255.0f * sx);
                                    u = sk1 * fmaf(16777216.0f, uraw, -255.0f * sx);
                                }
                                if (args.raw_gu) {
                                    args.out[(size_t)route * 2 * L.F + f] = g;
                                    args.out[((size_t)route * 2 + 1) * L.F + f] = u;
                                } else {
                                    args.out[(size_t)route * L.F + f] = silu_f32(g) * u;
                                }
                            }
                        }
                    } else {
                        const int d = mtile * kGBM + row;
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const int col = c0 + c;
                            if (col < n) {
                                float yv;
                                if constexpr (FP8) yv = (sk0 * rsc[c].y) * __uint_as_float(v[c]);
                                else yv = (sk0 * rsc[c].y) * fmaf(16777216.0f, __uint_as_float(v[c]), -255.0f * rsc[c].x);
                                args.out[(size_t)(r0 + n0 + col) * L.D + d] = yv;
                            }
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_d, kGTmemCols);
    }
}

// ------------------------------------------------------------------------------ helpers

// Route-ordered fp16 activation rows, one warp per destination row j: the source row is
// perm[j] / k (the token of grouped route j) or j itself when perm is null; ROTATE
// applies the 128-wide rotation on the way.  rowsum[j] = fp32 sum of the stored fp16
// values.  With rowscale (the rotated h rows of the down projection) the row is stored
// as v / 2^e, 2^e = rowscale[j] chosen so that its largest magnitude lies in
// [2^14, 2^15) (2^e = 1 for a zero row, 2^e >= 2^-112); a row of at most KEPT * 128
// values stays in registers between the max and the store pass, a longer one is read
// twice.  An out-of-range source raises device flag bit 0 and stores zeros.
constexpr int kRowsKept = 8;   // 128-value chunks per lane kept in registers (rows of <= 1024)

template <typename T, bool ROTATE>
__global__ void __launch_bounds__(256) route_rows_kernel(const T *__restrict__ x, int dst_rows, int cols,
                                                         const int32_t *__restrict__ perm, int k, int src_rows,
                                                         __half *__restrict__ dst, float *__restrict__ rowsum,
                                                         float *__restrict__ rowscale) {
    const int j = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (j >= dst_rows) return;
    const int src = perm ? perm[j] / k : j;
    const bool valid = src >= 0 && src < src_rows && (!perm || perm[j] >= 0);
    if (!valid && lane == 0) raise_flag(1);
    auto load = [&](int c, float (&v)[4]) {
        v[0] = v[1] = v[2] = v[3] = 0.f;
        if (valid) {
            float4 f = load4<T>(x + (size_t)src * cols + c + 4 * lane);
            v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
            if (ROTATE) fwht128_warp(v, lane);
        }
    };
    const bool keep = rowscale && cols <= kRowsKept * 128;
    float kept[kRowsKept][4];
    float inv_scale = 1.f;
    if (rowscale) {
        float m = 0.f;
        if (keep) {
#pragma unroll
            for (int q = 0; q < kRowsKept; ++q)
                if (q * 128 < cols) {
                    load(q * 128, kept[q]);
                    m = fmaxf(fmaxf(fabsf(kept[q][0]), fabsf(kept[q][1])),
                              fmaxf(fmaxf(fabsf(kept[q][2]), fabsf(kept[q][3])), m));
                }
        } else {
            for (int c = 0; c < cols; c += 128) {
                float v[4];
                load(c, v);
                m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fmaxf(fabsf(v[2]), fabsf(v[3])), m));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const int e = m > 0.f ? max(ilogbf(m) - 14, -112) : 0;   // 2^e and 2^-e stay normal
        inv_scale = ldexpf(1.f, -e);
        if (lane == 0) rowscale[j] = ldexpf(1.f, e);
    }
    float sum = 0.f;
    auto store = [&](int c, const float (&v)[4]) {
        __half2 lo = __floats2half2_rn(v[0] * inv_scale, v[1] * inv_scale);
        __half2 hi = __floats2half2_rn(v[2] * inv_scale, v[3] * inv_scale);
        const float2 lf = __half22float2(lo), hf = __half22float2(hi);
        sum += (lf.x + lf.y) + (hf.x + hf.y);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t *>(&lo);
        u.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(dst + (size_t)j * cols + c + 4 * lane) = u;
    };
    if (keep) {
#pragma unroll
        for (int q = 0; q < kRowsKept; ++q)
            if (q * 128 < cols) store(q * 128, kept[q]);
    } else {
        for (int c = 0; c < cols; c += 128) {
            float v[4];
            load(c, v);
            store(c, v);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) rowsum[j] = sum;
}

// The two-sided transform between the gate/up and down GEMMs, one warp per route row j:
// g = sign_gu * rotate(g), u likewise (the output side of gate and up), h = silu(g) * u,
// h' = rotate(sign_h * h) (the input side of down), stored fp16 as h' / rowscale[j] (the
// power of two that puts the row's largest magnitude in [2^14, 2^15)) with the fp32 sum
// of the stored values.  The row is computed twice (its maximum first).
__global__ void __launch_bounds__(256) swiglu_rows_kernel(const float *__restrict__ gu, int rows, int F,
                                                          const int8_t *__restrict__ sign_gu,
                                                          const int8_t *__restrict__ sign_h, __half *__restrict__ dst,
                                                          float *__restrict__ rowsum, float *__restrict__ rowscale) {
    const int j = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (j >= rows) return;
    auto row_chunk = [&](int c, float (&h)[4]) {
        const float4 g4 = load4<float>(gu + (size_t)j * 2 * F + c + 4 * lane);
        const float4 u4 = load4<float>(gu + ((size_t)j * 2 + 1) * F + c + 4 * lane);
        float g[4] = {g4.x, g4.y, g4.z, g4.w}, u[4] = {u4.x, u4.y, u4.z, u4.w};
        fwht128_warp(g, lane);
        fwht128_warp(u, lane);
        const char4 so = *reinterpret_cast<const char4 *>(sign_gu + c + 4 * lane);
        const char4 si = *reinterpret_cast<const char4 *>(sign_h + c + 4 * lane);
        const float o[4] = {(float)so.x, (float)so.y, (float)so.z, (float)so.w};
        const float in[4] = {(float)si.x, (float)si.y, (float)si.z, (float)si.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = silu_f32(g[i] * o[i]) * (u[i] * o[i]) * in[i];
        fwht128_warp(h, lane);
    };
    float m = 0.f;
    for (int c = 0; c < F; c += 128) {
        float h[4];
        row_chunk(c, h);
        m = fmaxf(fmaxf(fabsf(h[0]), fabsf(h[1])), fmaxf(fmaxf(fabsf(h[2]), fabsf(h[3])), m));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int e = m > 0.f ? max(ilogbf(m) - 14, -112) : 0;   // 2^e and 2^-e stay normal
    const float inv_scale = ldexpf(1.f, -e);
    if (lane == 0) rowscale[j] = ldexpf(1.f, e);
    float sum = 0.f;
    for (int c = 0; c < F; c += 128) {
        float h[4];
        row_chunk(c, h);
        __half2 lo = __floats2half2_rn(h[0] * inv_scale, h[1] * inv_scale);
        __half2 hi = __floats2half2_rn(h[2] * inv_scale, h[3] * inv_scale);
        const float2 lf = __half22float2(lo), hf = __half22float2(hi);
        sum += (lf.x + lf.y) + (hf.x + hf.y);
        uint2 w;
        w.x = *reinterpret_cast<uint32_t *>(&lo);
        w.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(dst + (size_t)j * F + c + 4 * lane) = w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) rowsum[j] = sum;
}

// E4M3 bytes of four floats (v[0] in the lowest byte), nearest even, saturating.
__device__ __forceinline__ uint32_t e4m3x4_from_f32(const float (&v)[4]) {
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(v[1]), "f"(v[0]));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(v[3]), "f"(v[2]));
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

// Power of two 2^e that puts a row's largest magnitude m in (224, 448] (E4M3's largest
// value is 448); 1 for a zero row.
__device__ __forceinline__ int e4m3_row_exponent(float m) {
    if (!(m > 0.f)) return 0;
    int e = ilogbf(m) - 8;                       // m / 2^e in [256, 512)
    if (ldexpf(m, -e) > 448.f) ++e;              // -> (224, 256)
    return max(e, -100);
}

// Route-ordered E4M3 activation rows for the pair-trellis GEMM, one warp per destination
// row j (source row perm[j] / k, or j when perm is null; ROTATE applies the 128-wide
// rotation): the row is scaled by 2^-e (e4m3_row_exponent of its largest magnitude),
// rounded to E4M3 and stored as bytes [j][cols]; rowscale[j] = 2^e.  The row is read twice.
// An out-of-range source raises device flag bit 0 and stores zeros.
template <typename T, bool ROTATE>
__global__ void __launch_bounds__(256) route_rows_e4m3_kernel(const T *__restrict__ x, int dst_rows, int cols,
                                                              const int32_t *__restrict__ perm, int k, int src_rows,
                                                              uint8_t *__restrict__ dst, float *__restrict__ rowscale) {
    const int j = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (j >= dst_rows) return;
    const int src = perm ? perm[j] / k : j;
    const bool valid = src >= 0 && src < src_rows && (!perm || perm[j] >= 0);
    if (!valid && lane == 0) raise_flag(1);
    auto load = [&](int c, float (&v)[4]) {
        v[0] = v[1] = v[2] = v[3] = 0.f;
        if (valid) {
            float4 f = load4<T>(x + (size_t)src * cols + c + 4 * lane);
            v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
            if (ROTATE) fwht128_warp(v, lane);
        }
    };
    // rows of at most kRowsKept * 128 values stay in registers between the two passes
    const bool keep = cols <= kRowsKept * 128;
    float kept[kRowsKept][4];
    float m = 0.f;
    if (keep) {
#pragma unroll
        for (int q = 0; q < kRowsKept; ++q)
            if (q * 128 < cols) {
                load(q * 128, kept[q]);
                m = fmaxf(fmaxf(fabsf(kept[q][0]), fabsf(kept[q][1])), fmaxf(fmaxf(fabsf(kept[q][2]), fabsf(kept[q][3])), m));
            }
    } else {
        for (int c = 0; c < cols; c += 128) {
            float v[4];
            load(c, v);
            m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fmaxf(fabsf(v[2]), fabsf(v[3])), m));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int e = e4m3_row_exponent(m);
    const float inv = ldexpf(1.f, -e);
    if (lane == 0) rowscale[j] = ldexpf(1.f, e);
    auto store = [&](int c, float (&v)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] *= inv;
        *reinterpret_cast<uint32_t *>(dst + (size_t)j * cols + c + 4 * lane) = e4m3x4_from_f32(v);
    };
    if (keep) {
#pragma unroll
        for (int q = 0; q < kRowsKept; ++q)
            if (q * 128 < cols) store(q * 128, kept[q]);
    } else {
        for (int c = 0; c < cols; c += 128) {
            float v[4];
            load(c, v);
            store(c, v);
        }
    }
}

// The two-sided transform between the pair-trellis GEMMs: as swiglu_rows_kernel, with
// h' stored as E4M3 bytes of h' / 2^e (e4m3_row_exponent) and rowscale[j] = 2^e.
__global__ void __launch_bounds__(256) swiglu_rows_e4m3_kernel(const float *__restrict__ gu, int rows, int F,
                                                               const int8_t *__restrict__ sign_gu,
                                                               const int8_t *__restrict__ sign_h,
                                                               uint8_t *__restrict__ dst, float *__restrict__ rowscale) {
    const int j = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (j >= rows) return;
    auto row_chunk = [&](int c, float (&h)[4]) {
        const float4 g4 = load4<float>(gu + (size_t)j * 2 * F + c + 4 * lane);
        const float4 u4 = load4<float>(gu + ((size_t)j * 2 + 1) * F + c + 4 * lane);
        float g[4] = {g4.x, g4.y, g4.z, g4.w}, u[4] = {u4.x, u4.y, u4.z, u4.w};
        fwht128_warp(g, lane);
        fwht128_warp(u, lane);
        const char4 so = *reinterpret_cast<const char4 *>(sign_gu + c + 4 * lane);
        const char4 si = *reinterpret_cast<const char4 *>(sign_h + c + 4 * lane);
        const float o[4] = {(float)so.x, (float)so.y, (float)so.z, (float)so.w};
        const float in[4] = {(float)si.x, (float)si.y, (float)si.z, (float)si.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = silu_f32(g[i] * o[i]) * (u[i] * o[i]) * in[i];
        fwht128_warp(h, lane);
    };
    float m = 0.f;
    for (int c = 0; c < F; c += 128) {
        float h[4];
        row_chunk(c, h);
        m = fmaxf(fmaxf(fabsf(h[0]), fabsf(h[1])), fmaxf(fmaxf(fabsf(h[2]), fabsf(h[3])), m));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int e = e4m3_row_exponent(m);
    const float inv = ldexpf(1.f, -e);
    if (lane == 0) rowscale[j] = ldexpf(1.f, e);
    for (int c = 0; c < F; c += 128) {
        float h[4];
        row_chunk(c, h);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] *= inv;
        *reinterpret_cast<uint32_t *>(dst + (size_t)j * F + c + 4 * lane) = e4m3x4_from_f32(h);
    }
}

// Tiles of <= 256 routes per active expert: out[0] = count, then (expert, first route).
__global__ void __launch_bounds__(1024) gemm_tile_list_kernel(const int32_t *__restrict__ offsets,
                                                              const int32_t *__restrict__ active_ids,
                                                              const int32_t *__restrict__ n_active_p, int max_tiles,
                                                              int32_t *__restrict__ out) {
    __shared__ int32_t warp_sum[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_active = *n_active_p;
    int running = 0;
    for (int base = 0; base < n_active; base += 1024) {
        const int a = base + tid;
        int e = -1, cnt = 0;
        if (a < n_active) {
            e = active_ids[a];
            cnt = (offsets[e + 1] - offsets[e] + kGBN - 1) / kGBN;
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_sum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int s = warp_sum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int v = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += v;
            }
            warp_sum[lane] = s;
        }
        __syncthreads();
        const int excl = running + (warp ? warp_sum[warp - 1] : 0) + incl - cnt;
        for (int i = 0; i < cnt; ++i) {
            const int ti = excl + i;
            if (ti < max_tiles) {
                out[1 + 2 * ti] = e;
                out[2 + 2 * ti] = i * kGBN;
            }
        }
        running += warp_sum[31];
        __syncthreads();
    }
    if (tid == 0) out[0] = min(running, max_tiles);
}

// ------------------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Route-ordered activations [rows][cols] (fp16, or E4M3 bytes) -> 4 maps with boxes of
// one 128-byte row segment (64 fp16 or 128 E4M3 columns) x {32, 64, 128, 256} rows and
// the 128-byte swizzle.
static int make_maps(const void *base, int rows, int cols, bool e4m3, GemmMaps &maps) {
    auto enc = tensor_map_encoder();
    if (!enc) return record_error("cuTensorMapEncodeTiled entry point not found");
    const size_t esize = e4m3 ? 1 : sizeof(__half);
    for (int b = 0; b < kGBoxes; ++b) {
        cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
        cuuint64_t strides[1] = {(cuuint64_t)cols * esize};
        cuuint32_t box[2] = {(cuuint32_t)(kGRowBytes / esize), (cuuint32_t)(32 << b)};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = enc(&maps.b[b], e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                         (void *)base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return record_error("cuTensorMapEncodeTiled failed");
    }
    return TQ_OK;
}

// Bit streams of every width group for one projection as a 3D uint32 tensor
// [n_experts][n_strips][words_per_strip], box {tiles_per_kb tiles, box_strips, 1}.
static int make_bits_maps(const tq_moe_layer *L, bool gateup, int tiles_per_kb, GemmMaps &maps) {
    auto enc = tensor_map_encoder();
    if (!enc) return record_error("cuTensorMapEncodeTiled entry point not found");
    for (int g = 0; g < 3; ++g) {
        for (int which = 0; which < 2; ++which) {
            CUtensorMap *dst = which ? &maps.bits_second[g] : &maps.bits_first[g];
            memset(dst, 0, sizeof(CUtensorMap));
            if (g >= L->n_groups || L->groups[g].n_experts == 0 || (!gateup && which)) continue;
            const tq_width_group &G = L->groups[g];
            const uint32_t *base = gateup ? (which ? G.up : G.gate) : G.down;
            const int n_strips = gateup ? L->F / 16 : L->D / 16;
            const int tiles = gateup ? L->D / 16 : L->F / 16;
            const cuuint64_t words = (cuuint64_t)tiles * 8 * G.K;
            cuuint64_t dims[3] = {words, (cuuint64_t)n_strips, (cuuint64_t)G.n_experts};
            cuuint64_t strides[2] = {words * 4, words * 4 * (cuuint64_t)n_strips};
            cuuint32_t box[3] = {(cuuint32_t)(tiles_per_kb * 8 * G.K), (cuuint32_t)(gateup ? 8 : 16), 1};
            cuuint32_t estr[3] = {1, 1, 1};
            CUresult r = enc(dst, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, (void *)base, dims, strides, box, estr,
                             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            if (r != CUDA_SUCCESS) return record_error("cuTensorMapEncodeTiled (bit streams) failed");
        }
    }
    return TQ_OK;
}

static size_t align256_g(size_t b) { return (b + 255) & ~(size_t)255; }

static int gemm_max_tiles(int T, int k, int E) {
    const long long routes = (long long)T * k;
    return (int)(routes / kGBN + min((long long)E, routes) + 1);
}

size_t gemm_workspace_bytes(const tq_moe_layer *L, int T, int k) {
    const size_t R = (size_t)T * k;
    const size_t hcols = L->sign_gu ? 2 : 1;   // two-sided: g and u, else h
    return align256_g(R * L->D * sizeof(__half)) + align256_g(R * sizeof(float)) +
           align256_g(R * hcols * L->F * sizeof(float)) + align256_g(R * L->F * sizeof(__half)) +
           align256_g(R * sizeof(float)) + align256_g(R * sizeof(float)) +
           align256_g((1 + 2 * (size_t)gemm_max_tiles(T, k, L->E)) * sizeof(int32_t));
}

template <bool FP8>
static int set_gemm_smem() {
    const int bytes = (int)(sizeof(GemmSmem) + 1024);
    if (cudaFuncSetAttribute(moe_gemm_kernel<true, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(moe_gemm_kernel<false, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
            cudaSuccess)
        return record_cuda_error("cudaFuncSetAttribute(moe_gemm_kernel)");
    return TQ_OK;
}

// The routed experts through the tensor-core GEMM.  Workspace: route-ordered activation
// rows (fp16 for T16; E4M3 bytes for the pair trellis) and one float per route (T16: the
// row sum; pair trellis: the row's power-of-two scale), h (or g and u when two-sided),
// the rotated h' rows (fp16 h' / 2^e, or E4M3), their row sums and scales, the tile list.
int run_moe_gemm(const tq_moe_layer *L, const __half *x_rot, const int32_t *offsets, const int32_t *perm,
                 const int32_t *active_ids, const int32_t *n_active, int T, int k, float *y_perm, void *ws,
                 cudaStream_t s) {
    static PerDeviceFlag configured;
    if (!configured.get()) {
        if (set_gemm_smem<false>() || set_gemm_smem<true>()) return TQ_ERR_CUDA;
        configured.set();
    }
    const bool fp8 = L->codebook == TQ_CODEBOOK_PAIR_E4M3;
    const int R = T * k;
    char *w = reinterpret_cast<char *>(ws);
    void *xp = w;
    w += align256_g((size_t)R * L->D * sizeof(__half));
    float *sxp = reinterpret_cast<float *>(w);   // T16: row sums of x'; pair trellis: row scales
    w += align256_g((size_t)R * sizeof(float));
    const int two = L->sign_gu != nullptr;     // two-sided transform
    float *h = reinterpret_cast<float *>(w);   // h, or g and u when two-sided
    w += align256_g((size_t)R * (two ? 2 : 1) * L->F * sizeof(float));
    void *hr = w;
    w += align256_g((size_t)R * L->F * sizeof(__half));
    float *shr = reinterpret_cast<float *>(w);
    w += align256_g((size_t)R * sizeof(float));
    float *scr = reinterpret_cast<float *>(w);   // power-of-two scale of each h' row
    w += align256_g((size_t)R * sizeof(float));
    int32_t *tiles = reinterpret_cast<int32_t *>(w);
    const int max_tiles = gemm_max_tiles(T, k, L->E);

    GemmMaps maps_x, maps_h;
    int st = make_maps(xp, R, L->D, fp8, maps_x);
    if (st) return st;
    st = make_maps(hr, R, L->F, fp8, maps_h);
    if (st) return st;
    const int tiles_per_kb = fp8 ? GemmShape<true>::kTiles : GemmShape<false>::kTiles;
    st = make_bits_maps(L, true, tiles_per_kb, maps_x);
    if (st) return st;
    st = make_bits_maps(L, false, tiles_per_kb, maps_h);
    if (st) return st;

    const size_t smem = sizeof(GemmSmem) + 1024;
    const unsigned row_blocks = (unsigned)(((size_t)R * 32 + 255) / 256);
    {
        LaunchScope ls(s, kStageGemmPrep);
        gemm_tile_list_kernel<<<1, 1024, 0, s>>>(offsets, active_ids, n_active, max_tiles, tiles);
    }
    st = launch_status();
    if (st) return st;
    {
        // x_rot is already rotated: copy its rows to their route rows (+ row sums, or as
        // scaled E4M3)
        LaunchScope ls(s, kStageGemmPrep);
        if (fp8)
            route_rows_e4m3_kernel<__half, false><<<row_blocks, 256, 0, s>>>(x_rot, R, L->D, perm, k, T,
                                                                            reinterpret_cast<uint8_t *>(xp), sxp);
        else
            route_rows_kernel<__half, false><<<row_blocks, 256, 0, s>>>(x_rot, R, L->D, perm, k, T,
                                                                       reinterpret_cast<__half *>(xp), sxp, nullptr);
    }
    st = launch_status();
    if (st) return st;
    {
        const dim3 grid(L->F / (64 * kGTiles), max_tiles);
        LaunchScope ls(s, kStageGemmGateUp);
        if (fp8) {
            GemmArgs a{*L, offsets, tiles, nullptr, sxp, h, L->D, two};
            moe_gemm_kernel<true, true><<<grid, kGThreads, smem, s>>>(maps_x, a);
        } else {
            GemmArgs a{*L, offsets, tiles, sxp, nullptr, h, L->D, two};
            moe_gemm_kernel<true, false><<<grid, kGThreads, smem, s>>>(maps_x, a);
        }
    }
    st = launch_status();
    if (st) return st;
    {
        LaunchScope ls(s, kStageRotateH);
        if (fp8) {
            uint8_t *h8 = reinterpret_cast<uint8_t *>(hr);
            if (two)
                swiglu_rows_e4m3_kernel<<<row_blocks, 256, 0, s>>>(h, R, L->F, L->sign_gu, L->sign_h, h8, scr);
            else
                route_rows_e4m3_kernel<float, true><<<row_blocks, 256, 0, s>>>(h, R, L->F, nullptr, 1, R, h8, scr);
        } else {
            __half *h16 = reinterpret_cast<__half *>(hr);
            if (two)
                swiglu_rows_kernel<<<row_blocks, 256, 0, s>>>(h, R, L->F, L->sign_gu, L->sign_h, h16, shr, scr);
            else
                route_rows_kernel<float, true><<<row_blocks, 256, 0, s>>>(h, R, L->F, nullptr, 1, R, h16, shr, scr);
        }
    }
    st = launch_status();
    if (st) return st;
    {
        const dim3 grid(L->D / (kGBM * kGTiles), max_tiles);
        LaunchScope ls(s, kStageGemmDown);
        if (fp8) {
            GemmArgs a{*L, offsets, tiles, nullptr, scr, y_perm, L->F, 0};
            moe_gemm_kernel<false, true><<<grid, kGThreads, smem, s>>>(maps_h, a);
        } else {
            GemmArgs a{*L, offsets, tiles, shr, scr, y_perm, L->F, 0};
            moe_gemm_kernel<false, false><<<grid, kGThreads, smem, s>>>(maps_h, a);
        }
    }
    return launch_status();
}

}  // namespace tq

int moe_validate_call(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                      const int32_t *perm, const int32_t *active_ids, const int32_t *n_active, int T,
                      int k, float *y_perm, void *ws, size_t ws_bytes);

TQ_API int moe_trellis_gemm(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                            const int32_t *perm, const int32_t *active_ids, const int32_t *n_active, int T,
                            int k, float *y_perm, void *ws, size_t ws_bytes, tq_stream stream) {
    int st = moe_validate_call(layer, x_rot, offsets, perm, active_ids, n_active, T, k, y_perm, ws, ws_bytes);
    if (st || T == 0) return st;
    if (ws_bytes < tq::gemm_workspace_bytes(layer, T, k)) return TQ_ERR_WORKSPACE;
    if (layer->D % (tq::kGBM * tq::kGTiles)) return TQ_ERR_UNSUPPORTED;   // down: 256-row CTAs
    if ((long long)T * k / tq::kGBN + layer->E + 1 > 65535) return TQ_ERR_UNSUPPORTED;
    return tq::run_moe_gemm(layer, reinterpret_cast<const __half *>(x_rot), offsets, perm, active_ids, n_active,
                            T, k, y_perm, ws, (cudaStream_t)stream);
}
