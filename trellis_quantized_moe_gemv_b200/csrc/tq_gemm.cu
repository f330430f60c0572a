// Prefill-sized routed-expert GEMM on tcgen05 tensor cores.
//
// Not implemented yet in this build: the entry point validates its arguments and
// returns TQ_ERR_UNSUPPORTED, so callers fail loudly instead of getting a result from
// another path.
#include "tq_common.cuh"

int moe_validate_call(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                      const int32_t *perm, const int32_t *active_ids, const int32_t *n_active, int T,
                      int k, float *y_perm, void *ws, size_t ws_bytes);

TQ_API int moe_trellis_gemm(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                            const int32_t *perm, const int32_t *active_ids, const int32_t *n_active, int T,
                            int k, float *y_perm, void *ws, size_t ws_bytes, tq_stream stream) {
    (void)stream;
    int st = moe_validate_call(layer, x_rot, offsets, perm, active_ids, n_active, T, k, y_perm, ws, ws_bytes);
    if (st || T == 0) return st;
    return TQ_ERR_UNSUPPORTED;
}
