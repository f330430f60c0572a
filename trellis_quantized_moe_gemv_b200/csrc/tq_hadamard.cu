// 128-wide Hadamard rotation of activations ("128-wide Hadamard rotations", dsx T16
// card, "How T16 works"; its "warp Hadamard transforms", "October 25 runtime
// checkpoint"): x'_chunk = (1/sqrt(128)) * H_128 x_chunk with H_128 the natural-order
// Sylvester matrix, i.e. butterflies over the 7 index bits.
//
// One warp per 128-chunk.  Lane l holds elements 4l..4l+3: index bits 0 and 1 are
// butterflies inside the lane, bits 2..6 pair lane l with lane l ^ (1 << (b-2)).
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

template <typename T>
__global__ void __launch_bounds__(256) hadamard128_kernel(const T *__restrict__ x, long long n_chunks,
                                                          __half *__restrict__ out) {
    const long long chunk = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (chunk >= n_chunks) return;
    const size_t off = (size_t)chunk * 128 + 4 * lane;
    float4 f = load4<T>(x + off);
    float v[4] = {f.x, f.y, f.z, f.w};
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
                       cudaStream_t s, int stage) {
    const long long n_chunks = rows * (cols / 128);
    if (n_chunks == 0) return TQ_OK;
    const int threads = 256;
    const long long blocks = (n_chunks * 32 + threads - 1) / threads;
    if (blocks > 0x7fffffffll) return TQ_ERR_UNSUPPORTED;
    LaunchScope ls(s, stage);
    switch (x_dtype) {
        case TQ_DTYPE_F16:
            hadamard128_kernel<__half><<<(unsigned)blocks, threads, 0, s>>>((const __half *)x, n_chunks, out);
            break;
        case TQ_DTYPE_BF16:
            hadamard128_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, s>>>(
                (const __nv_bfloat16 *)x, n_chunks, out);
            break;
        case TQ_DTYPE_F32:
            hadamard128_kernel<float><<<(unsigned)blocks, threads, 0, s>>>((const float *)x, n_chunks, out);
            break;
        default:
            return TQ_ERR_INVALID_ARG;
    }
    return launch_status();
}

}  // namespace tq

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
