// Shared device/host helpers of the sm_100a trellis-MoE library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <utility>

#include "trellis_moe.h"

#define TQ_API extern "C" __attribute__((visibility("default")))

namespace tq {

// T16 codebook multiplier ("How T16 works", item 1 of the dsx T16 card).
constexpr uint32_t kT16Mult = 0x3A2Fu;
// Decoded codes are t - 255 with t = byte0 + byte1 of the product.
constexpr int kCentre = 255;
// Fixed normaliser of every code: W = s * 2^-12 * c.
constexpr float kKappa = 1.0f / 4096.0f;
constexpr float kInvSqrt128 = 0.08838834764831845f;

// Device flag word (bit 0: bad id skipped, bit 1: bounded wait gave up).  The library
// is one translation unit (tq_library.cu), so this is its only definition.
__device__ int32_t g_device_flags = 0;

__device__ __forceinline__ void raise_flag(int32_t bit) { atomicOr(&g_device_flags, bit); }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned8(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

// ---------------------------------------------------------------------------- profiling
// Stage tags of the library's kernel launches (tq_profile_* in the C ABI).
enum Stage {
    kStageTopk = 0, kStagePermute = 1, kStageRotateX = 2, kStageMoeGemv = 3,
    kStageRotateH = 4, kStageGemvDown = 5, kStageUnpermute = 6, kStageDecode = 7,
    kStageGemv = 8, kStageGemmGateUp = 9, kStageGemmDown = 10, kStageGemmPrep = 11,
    kStageGemvQuant = 12, kStageEncode = 13, kStageGather = 14, kNumStages = 15
};

// Brackets one kernel launch: counts it and, while profiling is on, records a start
// and a stop event on the launching stream under the given stage tag.
struct LaunchScope {
    LaunchScope(cudaStream_t s, int stage);
    ~LaunchScope();
    cudaStream_t stream;
    int slot;
};

// Text of the most recent CUDA failure seen by the library (tq_last_error_string).
int record_error(const char *what);
int record_cuda_error(const char *what);

// Chained launches (programmatic dependent launch).  A kernel started by
// launch_chained may begin while the previous kernel on its stream is still finishing;
// its first statement is chain_entry(), which waits for that kernel to complete and
// its writes to be visible (so nothing another kernel wrote is read earlier than with a
// plain launch) and lets the next chained kernel be launched.  Both instructions do
// nothing in a kernel launched the ordinary way.
__device__ __forceinline__ void chain_entry() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                  Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline int launch_status() {
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) return TQ_OK;
    return record_error(cudaGetErrorString(e));
}

// Per-device caches: a process that drives several GPUs configures and sizes each one
// (kernel attributes apply to the current device); a device id past kMaxDevices is
// simply never cached.
constexpr int kMaxDevices = 64;
inline int current_device() {
    int d = 0;
    cudaGetDevice(&d);
    return d;
}
struct PerDeviceFlag {
    bool done[kMaxDevices] = {};
    bool get() const {
        const int d = current_device();
        return d >= 0 && d < kMaxDevices && done[d];
    }
    void set() {
        const int d = current_device();
        if (d >= 0 && d < kMaxDevices) done[d] = true;
    }
};

inline int num_sms() {
    static int cached[kMaxDevices] = {};
    const int dev = current_device();
    int n = dev >= 0 && dev < kMaxDevices ? cached[dev] : 0;
    if (n == 0) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
        if (dev >= 0 && dev < kMaxDevices) cached[dev] = n;
    }
    return n;
}

// ---------------------------------------------------------------------------- PTX wrappers

// Low 32 bits of the 64-bit value (hi:lo) >> sh, sh in [0, 31].
__device__ __forceinline__ uint32_t funnel_r(uint32_t lo, uint32_t hi, uint32_t sh) {
    return __funnelshift_r(lo, hi, sh);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// D = A * B + D,  m16n8k16, fp16 operands, fp32 accumulators (mma.sync register operands).
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------- mbarrier + bulk copy

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the asynchronous (bulk-copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before later
// asynchronous-proxy writes (a bulk copy refilling a buffer that was just read).
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16),
// completing `bytes` transaction bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, giving up after a bounded
// number of polls (each poll may suspend the thread for a hardware-defined time).
// Returns false (and raises device flag bit 1) if the wait gave up.
constexpr uint32_t kWaitPolls = 1u << 22;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitPolls; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    raise_flag(2);
    return false;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity, letting the hardware suspend the thread
// between polls (no spinning that would take issue slots from working warps), and give
// up after limit_ns of wall time (device flag bit 1).  Each poll may suspend for up to
// limit_ns / 256 (at most 1 ms); the timer is read every 8 polls.
constexpr uint64_t kWaitNs = 4000000000ull;
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t *bar, uint32_t parity, uint64_t limit_ns = kWaitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    const uint64_t h = limit_ns / 256;
    const uint32_t hint_ns = h > 1000000ull ? 1000000u : (h < 1000ull ? 1000u : (uint32_t)h);
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait_suspend(bar, parity, hint_ns)) return true;
        if ((n & 7u) == 0 && global_timer_ns() - t0 > limit_ns) break;
    }
    raise_flag(2);
    return false;
}

__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + expf(-z)); }

// ---------------------------------------------------------------------------- pair trellis
// The exlr8 card's pmcgx codebook ("Stores"): two weights share a 20-bit state (pair q of
// a tile reads stream bits 2Kq .. 2Kq + 19, tail-biting), each weight is the binary16 sum
// of the two halves of the state's product with its multiplier (mod 2^32), bit 14 of
// each half cleared, rounded to E4M3 (nearest even).  Pair q holds tile positions 2q and
// 2q + 1, i.e. rows 2(q mod 8) and 2(q mod 8) + 1 of column q div 8.
constexpr uint32_t kPairMultA = 0xCBAC1FEDu;
constexpr uint32_t kPairMultB = 0xBCA14C51u;
constexpr uint32_t kPairHalfMask = 0xBFFFBFFFu;   // bit 14 of both halves
constexpr float kKappa8 = 1.0f / 32.0f;           // W = s * 2^-5 * w

__device__ __forceinline__ uint32_t hadd2_rn(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// E4M3 bytes of two binary16 values (x: low half -> low byte), nearest even, saturating.
__device__ __forceinline__ uint32_t e4m3x2_from_f16x2(uint32_t x) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(d) : "r"(x));
    return d;
}

// 20-bit state of the pair whose window starts at compile-time bit offset O of v.
template <int O, int NS>
__device__ __forceinline__ uint32_t pair_state(const uint32_t (&v)[NS]) {
    constexpr int wi = O >> 5, sh = O & 31;
    const uint32_t x = sh == 0 ? v[wi] : funnel_r(v[wi], v[wi + 1], sh);
    return x & 0xFFFFFu;
}

// E4M3 bytes of one weight for two pairs (columns c0, c1 of the same row): P0, P1 are the
// two pairs' products with the weight's multiplier; the result's low byte is P0's weight.
__device__ __forceinline__ uint32_t pair_weights_e4m3x2(uint32_t P0, uint32_t P1) {
    const uint32_t lo = prmt(P0, P1, 0x5410u) & kPairHalfMask;   // {lo16(P0), lo16(P1)}
    const uint32_t hi = prmt(P0, P1, 0x7632u) & kPairHalfMask;   // {hi16(P0), hi16(P1)}
    return e4m3x2_from_f16x2(hadd2_rn(lo, hi));
}

// One lane cell of a tile: 16 rows x 4 consecutive columns (quarter t4: columns 4t4 ..
// 4t4 + 3, i.e. pairs 32 t4 .. 32 t4 + 31).  v holds the 2K words of the quarter's
// stream bits and the next word (tail-biting).  Writes the E4M3 bytes of row r, columns
// 4t4 .. 4t4 + 3 (byte c = column 4t4 + c) to rows[r].
template <int K, int I>
__device__ __forceinline__ void pair_cell_rows(const uint32_t (&v)[2 * K + 1], uint32_t (&rows)[16]) {
    if constexpr (I < 8) {
        uint32_t pa[4], pb[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            // pair 8c + I of the quarter starts at bit 2K (8c + I) of the lane's words
            const uint32_t st = c == 0 ? pair_state<2 * K * I>(v)
                              : c == 1 ? pair_state<2 * K * (8 + I)>(v)
                              : c == 2 ? pair_state<2 * K * (16 + I)>(v)
                                       : pair_state<2 * K * (24 + I)>(v);
            pa[c] = st * kPairMultA;
            pb[c] = st * kPairMultB;
        }
        rows[2 * I] = prmt(pair_weights_e4m3x2(pa[0], pa[1]), pair_weights_e4m3x2(pa[2], pa[3]), 0x5410u);
        rows[2 * I + 1] = prmt(pair_weights_e4m3x2(pb[0], pb[1]), pair_weights_e4m3x2(pb[2], pb[3]), 0x5410u);
        pair_cell_rows<K, I + 1>(v, rows);
    }
}

}  // namespace tq
