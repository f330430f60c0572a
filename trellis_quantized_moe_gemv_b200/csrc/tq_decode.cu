// Standalone T16 decode of a trellis-coded matrix to dense fp16 codes ("fixed-bit
// weight expansion", dsx T16 card, "October 25 runtime checkpoint"; codebook and
// column-major tiles, "How T16 works", items 1 and 2).
//
// A CTA covers one 16-row strip and up to 16 column tiles.  Thread (tile j, column q)
// decodes the 16 windows that run down column q: window (row r, column q) starts at
// stream bit 16Kq + Kr, so a thread's windows are one contiguous bit range.  Codes go
// through shared memory so that the global stores are whole 16-byte row segments.
#include "tq_common.cuh"

namespace tq {

constexpr int kDecTilesPerCta = 16;

template <int K>
__global__ void __launch_bounds__(256) trellis_decode_kernel(const uint32_t *__restrict__ bits,
                                                             int rows, int cols,
                                                             __half *__restrict__ out) {
    constexpr int WPT = 8 * K;                        // words per tile
    constexpr int SPAN_BITS = 15 * K + 16;            // bits covering 16 windows
    constexpr int NV = (SPAN_BITS + 31) / 32;         // normalised words
    __shared__ __align__(16) __half tile_codes[16][kDecTilesPerCta * 16 + 8];

    const int strip = blockIdx.y;
    const int tiles_per_row = cols / 16;
    const int j0 = blockIdx.x * kDecTilesPerCta;
    const int nt = min(kDecTilesPerCta, tiles_per_row - j0);
    const int jl = threadIdx.x >> 4;   // tile within the CTA
    const int q = threadIdx.x & 15;    // column within the tile

    if (jl < nt) {
        const uint32_t *tile = bits + ((size_t)strip * tiles_per_row + j0 + jl) * WPT;
        const int bit0 = 16 * K * q;
        const int w0 = bit0 >> 5;
        const int sh0 = bit0 & 31;     // 0, or 16 for odd columns at K = 3
        uint32_t raw[NV + 1];
#pragma unroll
        for (int i = 0; i <= NV; ++i) raw[i] = __ldg(tile + (w0 + i) % WPT);
        uint32_t v[NV + 1];
#pragma unroll
        for (int i = 0; i < NV; ++i) v[i] = funnel_r(raw[i], raw[i + 1], sh0);
        v[NV] = 0;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int o = K * r;
            const int wi = o >> 5, sh = o & 31;
            uint32_t win = sh == 0 ? v[wi] : funnel_r(v[wi], v[wi + 1], sh);
            uint32_t P = (win * kT16Mult) & 0xFFFFu;
            int t = (int)(P & 0xFFu) + (int)(P >> 8);
            tile_codes[r][jl * 16 + q] = __int2half_rn(t - kCentre);
        }
    }
    __syncthreads();
    // row-segment stores: 16 rows x (nt*16) fp16, 8 fp16 per 16-byte store
    const int segs_per_row = nt * 2;
    for (int s = threadIdx.x; s < 16 * segs_per_row; s += blockDim.x) {
        const int r = s / segs_per_row, c = (s % segs_per_row) * 8;
        uint4 val = *reinterpret_cast<const uint4 *>(&tile_codes[r][c]);
        *reinterpret_cast<uint4 *>(out + (size_t)(strip * 16 + r) * cols + j0 * 16 + c) = val;
    }
}

// Standalone decode of a pair-trellis (E4M3) matrix: thread (tile, quarter t4) decodes the
// 32 pairs of columns 4t4 .. 4t4 + 3 of its tile (pair_cell_rows) and stores each row's 4
// bytes.  out is E4M3 bytes [rows][cols], row-major.
template <int K>
__global__ void __launch_bounds__(256) trellis_decode_e4m3_kernel(const uint32_t *__restrict__ bits, int rows,
                                                                  int cols, uint8_t *__restrict__ out) {
    const int tiles_per_row = cols / 16;
    const long long n_cells = (long long)(rows / 16) * tiles_per_row * 4;
    const long long cell = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (cell >= n_cells) return;
    const int t4 = (int)(cell & 3);
    const long long tile = cell >> 2;
    const int strip = (int)(tile / tiles_per_row), tj = (int)(tile % tiles_per_row);
    const uint32_t *w = bits + (size_t)tile * (8 * K);
    uint32_t v[2 * K + 1];
#pragma unroll
    for (int i = 0; i < 2 * K; ++i) v[i] = __ldg(w + 2 * K * t4 + i);
    v[2 * K] = __ldg(w + 2 * K * ((t4 + 1) & 3));   // next quarter's first word (tail-biting)
    uint32_t r[16];
    pair_cell_rows<K, 0>(v, r);
#pragma unroll
    for (int i = 0; i < 16; ++i)
        *reinterpret_cast<uint32_t *>(out + (size_t)(strip * 16 + i) * cols + tj * 16 + 4 * t4) = r[i];
}

}  // namespace tq

TQ_API int trellis_decode_e4m3(const uint32_t *bits, int K, int rows, int cols, uint8_t *out, tq_stream stream) {
    if (K < 2 || K > 4 || rows < 0 || cols < 0 || rows % 16 || cols % 16) return TQ_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return TQ_OK;
    if (!bits || !out) return TQ_ERR_INVALID_ARG;
    if (!tq::aligned16(bits) || !tq::aligned16(out)) return TQ_ERR_ALIGNMENT;
    const long long cells = (long long)(rows / 16) * (cols / 16) * 4;
    if ((cells + 255) / 256 > 0x7fffffffll) return TQ_ERR_UNSUPPORTED;
    const unsigned grid = (unsigned)((cells + 255) / 256);
    cudaStream_t s = (cudaStream_t)stream;
    tq::LaunchScope ls(s, tq::kStageDecode);
    switch (K) {
        case 2: tq::trellis_decode_e4m3_kernel<2><<<grid, 256, 0, s>>>(bits, rows, cols, out); break;
        case 3: tq::trellis_decode_e4m3_kernel<3><<<grid, 256, 0, s>>>(bits, rows, cols, out); break;
        default: tq::trellis_decode_e4m3_kernel<4><<<grid, 256, 0, s>>>(bits, rows, cols, out); break;
    }
    return tq::launch_status();
}

TQ_API int trellis_decode(const uint32_t *bits, int K, int rows, int cols, uint16_t *out,
                          tq_stream stream) {
    if (K < 2 || K > 4 || rows < 0 || cols < 0 || rows % 16 || cols % 16) return TQ_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return TQ_OK;
    if (!bits || !out) return TQ_ERR_INVALID_ARG;
    if (!tq::aligned16(bits) || !tq::aligned16(out)) return TQ_ERR_ALIGNMENT;
    dim3 grid((cols / 16 + tq::kDecTilesPerCta - 1) / tq::kDecTilesPerCta, rows / 16);
    if (grid.y > 65535u) return TQ_ERR_UNSUPPORTED;
    cudaStream_t s = (cudaStream_t)stream;
    __half *o = reinterpret_cast<__half *>(out);
    tq::LaunchScope ls(s, tq::kStageDecode);
    switch (K) {
        case 2: tq::trellis_decode_kernel<2><<<grid, 256, 0, s>>>(bits, rows, cols, o); break;
        case 3: tq::trellis_decode_kernel<3><<<grid, 256, 0, s>>>(bits, rows, cols, o); break;
        default: tq::trellis_decode_kernel<4><<<grid, 256, 0, s>>>(bits, rows, cols, o); break;
    }
    return tq::launch_status();
}
