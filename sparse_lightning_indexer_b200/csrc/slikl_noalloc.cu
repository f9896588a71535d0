// slikl_grad_noalloc: the same computation as slikl_grad, for callers that cannot allocate
// device memory at call time (for example code running inside a memory pool that forbids
// cudaMalloc, or a runtime whose allocator is not reachable from the calling thread).
//
// The scratch memory that slikl_grad takes from the caller's workspace lives here in a fixed
// file-scope device array instead. Its size is fixed at build time (kNoAllocScratchBytes), it
// is created when the library's device code is loaded on a GPU and it stays allocated on every
// GPU that loaded the library until the process exits.
//
// Host code cannot pass the array's name to a kernel: on the host that name is only a
// stand-in object, not a device address. The device address is obtained once per device with
// cudaGetSymbolAddress while that device is current, checked, cached, and handed to
// slikl_grad as its workspace. That lookup happens on the first call on each device, so the
// first call on a device should not be made while a stream is being captured.
//
// All calls on one device share the array. slikl_grad clears what has to start at zero (the
// status word and the fp32 dk accumulator) at every call and rewrites the rest, so the
// contents left by an earlier call do not matter; two calls whose work overlaps on the GPU
// (different streams without ordering between them) race on the array and give wrong results.
#include <mutex>

#include "slikl_common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = SLIKL_NOALLOC_SCRATCH_BYTES;   // 32 MiB per GPU
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mutex;
void *g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" {

slikl_status slikl_grad_noalloc(const slikl_problem *problem, const slikl_tensors *tensors,
                                void *stream) {
    if (!problem) return SLIKL_ERR_PARAM_NULLPTR;
    if (problem->deterministic) return SLIKL_ERR_PARAM_INVALID;   // needs far more scratch
    // the scatter dK path: its scratch does not grow with the key range
    slikl_options opt{};
    opt.dk_path = SLIKL_DK_SCATTER;
    size_t need = 0;
    slikl_status st = slikl_grad_workspace_size_ex(problem, &opt, &need);
    if (st != SLIKL_OK) return st;
    if (need > kNoAllocScratchBytes) return SLIKL_ERR_WORKSPACE_TOO_SMALL;
    if (!tensors) return SLIKL_ERR_PARAM_NULLPTR;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SLIKL_ERR_CUDA;
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!g_scratch_addr[dev]) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
                return SLIKL_ERR_CUDA;
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    return slikl_grad_ex(problem, tensors, scratch, kNoAllocScratchBytes, stream, &opt);
}

}  // extern "C"
