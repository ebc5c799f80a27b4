// spffn_forward_noalloc: the neuron-aware FFN forward for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code running inside another
// allocator's arena, processes under a fixed device-memory budget, or callers
// that cannot provide the workspace an spffn_ctx needs.  This entry point takes
// only inputs and outputs; the fp32 partial sums of the split reduction live in
// a file-scope __device__ array that every GPU loading this library reserves
// once, until the process exits.
#include <mutex>
#include "spffn_internal.cuh"
#include "spffn_kernels.cuh"

namespace {

constexpr size_t kScratchBytes = (size_t)1 << 20;    // partial sums (1 MiB)
constexpr size_t kScratchCtl = 256;                   // error word (not reported by this entry point)
constexpr int kMaxDevices = 64;

// Shared by every call on a device; keeps the last call's contents.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes + kScratchCtl];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array for the current device (set up on the
// first call on that device, with that device current).
cudaError_t scratch_for_current_device(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" spffn_status spffn_forward_noalloc(const spffn_config* cfg, const spffn_weights* w, const void* x,
                                              int32_t B, const int32_t* idx, const int32_t* count, float* y,
                                              void* stream)
{
    if (!cfg || !w || !x || !idx || !count || !y) return SPFFN_ERR_INVALID_ARG;
    if (cfg->d < 64 || cfg->d > 16384 || cfg->d % 64 || cfg->n < 32 || cfg->n % 32 || cfg->n > 131072)
        return SPFFN_ERR_INVALID_ARG;
    if (cfg->dtype != SPFFN_F16 && cfg->dtype != SPFFN_BF16) return SPFFN_ERR_INVALID_ARG;
    if (B < 1 || B > spffn::kMaxPhaseBatch) return SPFFN_ERR_INVALID_ARG;
    if (!w->W1 || !w->b1 || !w->W2T) return SPFFN_ERR_INVALID_ARG;
    if (!aligned16(w->W1) || !aligned16(w->W2T) || !aligned16(x) || !aligned16(y)) return SPFFN_ERR_INVALID_ARG;
    // one partial sum is B x d fp32; at least one must fit the fixed scratch
    const size_t one = (size_t)B * cfg->d * sizeof(float);
    if (one > kScratchBytes) return SPFFN_ERR_UNSUPPORTED;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return SPFFN_ERR_CUDA;
    const int S = (int)std::min<size_t>((size_t)sms, kScratchBytes / one);
    void* base = nullptr;
    if (scratch_for_current_device(&base) != cudaSuccess) return SPFFN_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t* err = reinterpret_cast<uint32_t*>(static_cast<char*>(base) + kScratchBytes);
    if (cudaMemsetAsync(err, 0, sizeof(uint32_t), st) != cudaSuccess) return SPFFN_ERR_CUDA;
    cudaError_t e = spffn::launch_forward_scratch(*cfg, *w, x, B, idx, count, y, static_cast<float*>(base), S, err,
                                                  st);
    return e == cudaSuccess ? SPFFN_OK : SPFFN_ERR_CUDA;
}
