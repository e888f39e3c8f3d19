// nosa_noalloc.cu -- nosa_select_noalloc: nosa_select for callers that cannot
// allocate device memory.
//
// Who needs it: code that is handed only its inputs and outputs and has no way
// to obtain extra device memory -- for instance a plug-in running inside a
// host engine that owns the allocator and exposes none of it, or a latency-
// critical path that must not call cudaMalloc because cudaMalloc may
// synchronise the device.  Such a caller cannot provide the scratch workspace
// that nosa_select takes, so this entry point keeps that scratch in a fixed
// device array compiled into the library instead.
//
// The array is a file-scope __device__ array of NOSA_NOALLOC_SELECT_SCRATCH
// bytes.  Every GPU that loads the library holds it until the process exits.
// Host code cannot use the array's name as a device address, so the first call
// on each device resolves the address with cudaGetSymbolAddress (with that
// device current) and caches it.  The stream a call is given must belong to
// the current device, whose array address is the one passed to the kernel.
#include <mutex>
#include <string.h>

#include "nosa_internal.cuh"

namespace {

// Scratch of every nosa_select_noalloc call on a device: the per-unit
// completion counters followed by the per-chunk top-32 lists.
static __device__ __align__(256) uint8_t g_select_scratch[NOSA_NOALLOC_SELECT_SCRATCH];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_addr[kMaxDevices] = {};

// Device address of g_select_scratch on the current device (set up once per device).
int scratch_addr(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NOSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return NOSA_ERR_CUDA;
        }
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return NOSA_OK;
}

}  // namespace

extern "C" int nosa_select_noalloc(const nosa_config *cfg, const nosa_state *st, const uint16_t *q,
                                   int32_t *sel, int32_t *nsel, int32_t *gq, void *stream) {
    int rc = nosa_validate_config(cfg);
    if (rc) return rc;
    const size_t need = nosa_workspace_bytes(cfg, NOSA_WS_SELECT);
    if (need > NOSA_NOALLOC_SELECT_SCRATCH) return NOSA_ERR_CAPACITY;
    void *ws = nullptr;
    if (need > 0 && (rc = scratch_addr(&ws))) return rc;
    // every argument check of nosa_select runs before anything is queued on the stream
    if ((rc = nosa::select_args_ok(cfg, st, q, sel, nsel, gq, ws, need))) return rc;
    if (need > 0) {
        // the counters must start at zero; the lists are written before they are read
        const size_t counters = (size_t)cfg->batch * cfg->heads_kv * sizeof(int32_t);
        if (cudaMemsetAsync(ws, 0, counters, static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return NOSA_ERR_CUDA;
    }
    return nosa_select(cfg, st, q, sel, nsel, gq, ws, need, stream);
}

extern "C" int nosa_noalloc_scratch_poison(uint8_t byte, void *stream) {
    void *ws = nullptr;
    const int rc = scratch_addr(&ws);
    if (rc) return rc;
    return cudaMemsetAsync(ws, byte, NOSA_NOALLOC_SELECT_SCRATCH, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? NOSA_OK
               : NOSA_ERR_CUDA;
}
