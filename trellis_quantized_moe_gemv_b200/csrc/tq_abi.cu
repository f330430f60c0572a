// Status codes, version and the device anomaly flag word of the C ABI.
#include "tq_common.cuh"

#include <stdio.h>

TQ_API const char *tq_status_string(int status) {
    switch (status) {
        case TQ_OK: return "TQ_OK";
        case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG: invalid size, width, count or pointer";
        case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED: outside what this build implements";
        case TQ_ERR_ALIGNMENT: return "TQ_ERR_ALIGNMENT: pointer not aligned as documented";
        case TQ_ERR_WORKSPACE: return "TQ_ERR_WORKSPACE: workspace missing or too small";
        case TQ_ERR_CUDA: return "TQ_ERR_CUDA: CUDA launch or runtime error";
        case TQ_ERR_DEVICE_TIMEOUT: return "TQ_ERR_DEVICE_TIMEOUT: a bounded device wait gave up";
        default: return "unknown tq_status";
    }
}

TQ_API int tq_abi_version(void) { return TQ_ABI_VERSION; }

namespace tq {
static char g_last_error[256] = "";

int record_error(const char *what) {
    snprintf(g_last_error, sizeof(g_last_error), "%s", what ? what : "");
    return TQ_ERR_CUDA;
}

int record_cuda_error(const char *what) {
    cudaError_t e = cudaGetLastError();
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
    return TQ_ERR_CUDA;
}
}  // namespace tq

TQ_API const char *tq_last_error_string(void) { return tq::g_last_error; }

TQ_API int tq_device_status(int32_t *flags_out, int clear) {
    if (!flags_out) return TQ_ERR_INVALID_ARG;
    if (cudaMemcpyFromSymbol(flags_out, tq::g_device_flags, sizeof(int32_t)) != cudaSuccess)
        return TQ_ERR_CUDA;
    if (clear) {
        const int32_t zero = 0;
        if (cudaMemcpyToSymbol(tq::g_device_flags, &zero, sizeof(int32_t)) != cudaSuccess)
            return TQ_ERR_CUDA;
    }
    return TQ_OK;
}

// ---------------------------------------------------------------------------- profiling
namespace tq {

struct Profiler {
    bool on = false;
    uint32_t stage_mask = 0xFFFFFFFFu;   // stages whose launches are recorded
    int capacity = 0;
    int used = 0;
    cudaEvent_t *events = nullptr;   // 2 per recorded launch
    int *stage = nullptr;
};
static Profiler g_prof;
static unsigned long long g_launches = 0;

// Inside stream capture an event record becomes an external event-record node of the
// graph (re-recorded at every replay); otherwise it is an ordinary record.
static void record_event(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, s);
}

LaunchScope::LaunchScope(cudaStream_t s, int st) : stream(s), slot(-1) {
    ++g_launches;
    if (g_prof.on && g_prof.used < g_prof.capacity && st >= 0 && st < 32 && ((g_prof.stage_mask >> st) & 1u)) {
        slot = g_prof.used++;
        g_prof.stage[slot] = st;
        record_event(g_prof.events[2 * slot], s);
    }
}

LaunchScope::~LaunchScope() {
    if (slot >= 0) record_event(g_prof.events[2 * slot + 1], stream);
}

static void profile_release() {
    for (int i = 0; i < 2 * g_prof.capacity; ++i) cudaEventDestroy(g_prof.events[i]);
    delete[] g_prof.events;
    delete[] g_prof.stage;
    g_prof = Profiler();
}

}  // namespace tq

TQ_API unsigned long long tq_launch_count(void) { return tq::g_launches; }

TQ_API int tq_profile_enable(int max_launches) {
    if (max_launches < 1 || max_launches > (1 << 20)) return TQ_ERR_INVALID_ARG;
    tq::profile_release();
    tq::g_prof.events = new cudaEvent_t[2 * (size_t)max_launches];
    tq::g_prof.stage = new int[max_launches];
    for (int i = 0; i < 2 * max_launches; ++i) {
        if (cudaEventCreate(&tq::g_prof.events[i]) != cudaSuccess) {
            tq::g_prof.capacity = i / 2;
            tq::profile_release();
            return TQ_ERR_CUDA;
        }
    }
    tq::g_prof.capacity = max_launches;
    tq::g_prof.on = true;
    return TQ_OK;
}

TQ_API int tq_profile_stages(uint32_t stage_mask) {
    if (!tq::g_prof.on) return TQ_ERR_INVALID_ARG;
    tq::g_prof.stage_mask = stage_mask;
    return TQ_OK;
}

TQ_API int tq_profile_disable(void) {
    tq::profile_release();
    return TQ_OK;
}

TQ_API int tq_profile_collect(double *stage_ms, int32_t *stage_launches, int n_stages) {
    if (!stage_ms || !stage_launches || n_stages < 1) return TQ_ERR_INVALID_ARG;
    for (int i = 0; i < n_stages; ++i) {
        stage_ms[i] = 0.0;
        stage_launches[i] = 0;
    }
    if (!tq::g_prof.on) return TQ_OK;
    for (int l = 0; l < tq::g_prof.used; ++l) {
        if (cudaEventSynchronize(tq::g_prof.events[2 * l + 1]) != cudaSuccess) return TQ_ERR_CUDA;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, tq::g_prof.events[2 * l], tq::g_prof.events[2 * l + 1]) !=
            cudaSuccess) {
            cudaGetLastError();   // a captured launch whose graph was never replayed
            continue;
        }
        const int st = tq::g_prof.stage[l];
        if (st >= 0 && st < n_stages) {
            stage_ms[st] += ms;
            stage_launches[st] += 1;
        }
    }
    tq::g_prof.used = 0;
    return TQ_OK;
}

// ---------------------------------------------------------------------- failure check
namespace tq {
// One warp waits, with the library's bounded wait, for a phase of a fresh mbarrier that
// nothing ever arrives on: the wait gives up after limit_ns, raises device flag bit 1
// and the kernel returns normally.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    mbar_wait_sleep(&bar, 0, limit_ns);
}
}  // namespace tq

TQ_API int tq_selftest_bounded_wait(uint32_t limit_us, tq_stream stream) {
    if (limit_us < 1 || limit_us > 10000000u) return TQ_ERR_INVALID_ARG;
    tq::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_us * 1000ull);
    return tq::launch_status();
}
