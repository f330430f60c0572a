// 128-wide Hadamard rotation of activations ("128-wide Hadamard rotations", dsx T16
// card, "How T16 works"; its "warp Hadamard transforms", "October 25 runtime
// checkpoint"): x'_chunk = (1/sqrt(128)) * H_128 x_chunk with H_128 the natural-order
// Sylvester matrix, i.e. butterflies over the 7 index bits.
//
// One warp per 128-chunk.  Lane l holds elements 4l..4l+3: index bits 0 and 1 are
// butterflies inside the lane, bits 2..6 pair lane l with lane l ^ (1 << (b-2)).
#include "tq_combine.cuh"
#include "tq_common.cuh"

namespace tq {

template <typename T>
__device__ __forceinline__ float4 load4(const T *p);

template <>
__device__ __forceinline__ float4 load4<float>(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
}
template <>
__device__ __forceinline__ float4 load4<__half>(const __half *p) {
    uint2 u = *reinterpret_cast<const uint2 *>(p);
    float2 a = __half22float2(*reinterpret_cast<__half2 *>(&u.x));
    float2 b = __half22float2(*reinterpret_cast<__half2 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16 *p) {
    uint2 u = *reinterpret_cast<const uint2 *>(p);
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u.x));
    float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

// In-warp 128-point Walsh-Hadamard transform of v (lane holds 4 consecutive points),
// scaled by 1/sqrt(128).
__device__ __forceinline__ void fwht128_warp(float (&v)[4], int lane) {
    // bit 0
    float a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
    // bit 1
    v[0] = a0 + a2;
    v[2] = a0 - a2;
    v[1] = a1 + a3;
    v[3] = a1 - a3;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float p = __shfl_xor_sync(0xffffffffu, v[i], m);
            v[i] = upper ? (p - v[i]) : (v[i] + p);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] *= kInvSqrt128;
}

// signs (optional, int8 +1/-1 per column) multiply x before the rotation: the input
// side of the two-sided transform, x' = rotate(signs * x).
template <typename T>
__global__ void __launch_bounds__(256) hadamard128_kernel(const T *__restrict__ x, long long n_chunks,
                                                          const int8_t *__restrict__ signs, int chunks_per_row,
                                                          __half *__restrict__ out) {
    chain_entry();
    const long long chunk = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (chunk >= n_chunks) return;
    const size_t off = (size_t)chunk * 128 + 4 * lane;
    float4 f = load4<T>(x + off);
    float v[4] = {f.x, f.y, f.z, f.w};
    if (signs) {
        const int col = (int)(chunk % chunks_per_row) * 128 + 4 * lane;
        const char4 sg = *reinterpret_cast<const char4 *>(signs + col);
        v[0] *= sg.x; v[1] *= sg.y; v[2] *= sg.z; v[3] *= sg.w;
    }
    fwht128_warp(v, lane);
    __half2 lo = __floats2half2_rn(v[0], v[1]);
    __half2 hi = __floats2half2_rn(v[2], v[3]);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&lo);
    u.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(out + off) = u;
}

// Rotation launcher shared with the MoE path (rotating the SwiGLU activations h).
int launch_hadamard128(const void *x, int x_dtype, long long rows, long long cols, __half *out,
                       cudaStream_t s, int stage, const int8_t *signs = nullptr) {
    const long long n_chunks = rows * (cols / 128);
    if (n_chunks == 0) return TQ_OK;
    const int threads = 256;
    const long long blocks = (n_chunks * 32 + threads - 1) / threads;
    if (blocks > 0x7fffffffll) return TQ_ERR_UNSUPPORTED;
    LaunchScope ls(s, stage);
    switch (x_dtype) {
        case TQ_DTYPE_F16:
            launch_chained(hadamard128_kernel<__half>, (unsigned)blocks, threads, 0, s, (const __half *)x, n_chunks,
                           signs, (int)(cols / 128), out);
            break;
        case TQ_DTYPE_BF16:
            launch_chained(hadamard128_kernel<__nv_bfloat16>, (unsigned)blocks, threads, 0, s,
                           (const __nv_bfloat16 *)x, n_chunks, signs, (int)(cols / 128), out);
            break;
        case TQ_DTYPE_F32:
            launch_chained(hadamard128_kernel<float>, (unsigned)blocks, threads, 0, s, (const float *)x, n_chunks,
                           signs, (int)(cols / 128), out);
            break;
        default:
            return TQ_ERR_INVALID_ARG;
    }
    return launch_status();
}

// Combine with the output side of the two-sided transform of the down projection:
// out[t] = signs * rotate(sum_s w[t, s] * y_perm[inv[t*k + s]]), summed in slot order (the
// rotation is linear, so rotating once after the weighted sum equals rotating every
// route's output).  One warp per (token, 128-chunk).
__global__ void __launch_bounds__(256) route_unpermute_signed_kernel(
    const float *__restrict__ y_perm, const int32_t *__restrict__ inv, const float *__restrict__ w, int T, int k,
    int D, int n_routes, const int8_t *__restrict__ signs, float *__restrict__ out) {
    chain_entry();
    const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int chunks = D / 128;
    if (wid >= (long long)T * chunks) return;
    const int t = (int)(wid / chunks), c = (int)(wid % chunks);
    const int col = c * 128 + 4 * lane;
    const float4 a = combine_slots(y_perm, inv, w, t, k, D, n_routes, col, lane == 0);
    float v[4] = {a.x, a.y, a.z, a.w};
    fwht128_warp(v, lane);
    const char4 sg = *reinterpret_cast<const char4 *>(signs + col);
    *reinterpret_cast<float4 *>(out + (size_t)t * D + col) = make_float4(v[0] * sg.x, v[1] * sg.y, v[2] * sg.z, v[3] * sg.w);
}

}  // namespace tq

TQ_API int route_unpermute_signed(const float *y_perm, const int32_t *inv, const float *topk_w, int T, int k,
                                  int D, const int8_t *signs_y, float *out, tq_stream stream) {
    if (T < 0 || k < 1 || D < 128 || D % 128) return TQ_ERR_INVALID_ARG;
    if (T == 0) return TQ_OK;
    if (!y_perm || !inv || !topk_w || !out || !signs_y) return TQ_ERR_INVALID_ARG;
    if (!tq::aligned16(y_perm) || !tq::aligned16(out) || (reinterpret_cast<uintptr_t>(signs_y) & 3))
        return TQ_ERR_ALIGNMENT;
    cudaStream_t s = (cudaStream_t)stream;
    const long long warps = (long long)T * (D / 128);
    const long long blocks = (warps * 32 + 255) / 256;
    if (blocks > 0x7fffffffll) return TQ_ERR_UNSUPPORTED;
    tq::LaunchScope ls(s, tq::kStageUnpermute);
    tq::launch_chained(tq::route_unpermute_signed_kernel, (unsigned)blocks, 256, 0, s, y_perm, inv, topk_w, T, k, D,
                       T * k, signs_y, out);
    return tq::launch_status();
}

TQ_API int hadamard128_signed(const void *x, int x_dtype, int64_t rows, int64_t cols, const int8_t *signs,
                              uint16_t *out, tq_stream stream) {
    if (rows < 0 || cols < 0 || cols % 128) return TQ_ERR_INVALID_ARG;
    if (x_dtype != TQ_DTYPE_F16 && x_dtype != TQ_DTYPE_BF16 && x_dtype != TQ_DTYPE_F32)
        return TQ_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return TQ_OK;
    if (!x || !out || !signs) return TQ_ERR_INVALID_ARG;
    if (!tq::aligned16(x) || !tq::aligned16(out) || (reinterpret_cast<uintptr_t>(signs) & 3)) return TQ_ERR_ALIGNMENT;
    return tq::launch_hadamard128(x, x_dtype, rows, cols, reinterpret_cast<__half *>(out), (cudaStream_t)stream,
                                  tq::kStageRotateX, signs);
}

TQ_API int hadamard128(const void *x, int x_dtype, int64_t rows, int64_t cols, uint16_t *out,
                       tq_stream stream) {
    if (rows < 0 || cols < 0 || cols % 128) return TQ_ERR_INVALID_ARG;
    if (x_dtype != TQ_DTYPE_F16 && x_dtype != TQ_DTYPE_BF16 && x_dtype != TQ_DTYPE_F32)
        return TQ_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return TQ_OK;
    if (!x || !out) return TQ_ERR_INVALID_ARG;
    if (!tq::aligned16(x) || !tq::aligned16(out)) return TQ_ERR_ALIGNMENT;
    return tq::launch_hadamard128(x, x_dtype, rows, cols, reinterpret_cast<__half *>(out),
                                  (cudaStream_t)stream, tq::kStageRotateX);
}
