// as_linear_decode_noalloc: the decode entry point for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc: for example code running inside a
// host framework that owns all device memory through its own pool and
// forbids outside allocations, or a process that must stay within a fixed
// device-memory budget fixed at start-up.  For them this variant takes its
// scratch (split-K partial sums, per-slice arrival counters and, for top-k,
// the selection bitmask) from one file-scope device array instead of a
// caller-provided workspace.  The caller still passes inputs and outputs.
//
// The array is AS_NOALLOC_SCRATCH_BYTES long and every GPU that loads the
// library holds it until the process exits.  In host code the name of the
// array is only a host-side handle, not a device address, so the device
// address is fetched once per device with cudaGetSymbolAddress (with that
// device current) and cached; the first call on each device does this
// set-up, so it should be made before any stream capture.  The cached
// address belongs to the device's context: after cudaDeviceReset the
// module is loaded again and the array may move, so this entry point must
// not be called again in that process.  All calls share
// the array and it keeps the last call's contents: the part that must start
// at zero (the arrival counters) is cleared on the stream at every call, and
// calls whose executions overlap on the GPU race on the array.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace {

constexpr int AS_NOALLOC_MAX_DEVICES = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[AS_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[AS_NOALLOC_MAX_DEVICES] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device).
as_status noalloc_scratch(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return AS_ERR_CUDA;
    if (dev < 0 || dev >= AS_NOALLOC_MAX_DEVICES) return AS_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return AS_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return AS_OK;
}

}  // namespace

extern "C" as_status as_linear_decode_noalloc(const void *x, as_dtype dt, int T, int K, int n_out, const void *Wt,
                                              const float *g, const float *rowsum, const as_config *cfg, void *y,
                                              uint32_t *mask_out, float *eta_out, float *colnorm_out,
                                              cudaStream_t stream)
{
    // every argument is checked before the shared scratch is touched: a
    // refused call enqueues nothing on the stream
    as_status st = decode_check_args(x, dt, T, K, n_out, Wt, g, rowsum, cfg, y, mask_out, eta_out, colnorm_out);
    if (st != AS_OK) return st;
    const size_t need = as_workspace_size(AS_OP_DECODE, T, K, n_out, cfg);
    if (need == (size_t)-1) return AS_ERR_SHAPE;
    if (need > (size_t)AS_NOALLOC_SCRATCH_BYTES) return AS_ERR_WORKSPACE;
    void *scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != AS_OK) return st;
    // the arrival counters lead the scratch layout and must start at zero
    const as::DecodePlan plan = as::decode_plan(T, K, n_out, dt == AS_BF16);
    if (cudaMemsetAsync(scratch, 0, plan.counter_bytes, stream) != cudaSuccess) return AS_ERR_CUDA;
    return as_linear_decode(x, dt, T, K, n_out, Wt, g, rowsum, cfg, y, mask_out, eta_out, colnorm_out, scratch,
                            (size_t)AS_NOALLOC_SCRATCH_BYTES, stream);
}
