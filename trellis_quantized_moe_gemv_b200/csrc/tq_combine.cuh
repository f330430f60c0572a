// The weighted sum of the combine: out[t] = sum over slots s of w[t*k+s] * y_perm[inv[t*k+s]],
// added in slot order in fp32 (deterministic, no atomics).
#pragma once

#include "tq_common.cuh"

namespace tq {

// Four consecutive columns (col .. col+3) of token t's sum.  The routes' rows are loaded
// eight slots at a time before any of them is added, so their latencies overlap; the
// additions keep slot order.  A route index outside [0, n_routes) raises device flag
// bit 0 (from lanes with flag_lane set) and is skipped.
__device__ __forceinline__ float4 combine_slots(const float *__restrict__ y_perm, const int32_t *__restrict__ inv,
                                                const float *__restrict__ w, int t, int k, int D, int n_routes,
                                                int col, bool flag_lane) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < k; s0 += 8) {
        float4 y[8];
        float ws[8];
        bool ok[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int s = s0 + j;
            ok[j] = false;
            y[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            ws[j] = 0.f;
            if (s < k) {
                const int r = inv[t * k + s];
                ws[j] = w[t * k + s];
                ok[j] = r >= 0 && r < n_routes;
                if (ok[j])
                    y[j] = *reinterpret_cast<const float4 *>(y_perm + (size_t)r * D + col);
                else if (flag_lane)
                    raise_flag(1);
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (!ok[j]) continue;
            acc.x = fmaf(ws[j], y[j].x, acc.x);
            acc.y = fmaf(ws[j], y[j].y, acc.y);
            acc.z = fmaf(ws[j], y[j].z, acc.z);
            acc.w = fmaf(ws[j], y[j].w, acc.w);
        }
    }
    return acc;
}

}  // namespace tq
