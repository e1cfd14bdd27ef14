// ce_forward_noalloc: the row cross-entropy forward for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc or hand over a workspace: plugins that
// run inside a host application which owns every byte of the device through
// its own pool (a raw allocation would bypass its accounting or exceed its
// budget), loops with a fixed memory budget set at start-up that must not run
// out of memory halfway, and C callers with no allocator at hand (cudaMalloc
// may also synchronise the device, which a latency-bound caller cannot
// afford). The split-vocabulary forward needs scratch memory for its per-row
// partial states; this entry point takes that scratch from a fixed array in
// device memory that belongs to the library instead.
//
// The array is a file-scope __device__ variable of kScratchBytes bytes. Every
// device that loads the library holds one copy until the process exits.
// Host code cannot use the array's name as a device address (on the host it
// names a stand-in object), so the device address is looked up once per
// device with cudaGetSymbolAddress, with that device current, on the first
// call made on it, and cached; that first call on a device should come before
// any stream capture begins.
#include <mutex>

#include "ce_b200.h"

namespace {

constexpr size_t kScratchBytes = CE_NOALLOC_SCRATCH_BYTES;  // 64 KiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices];

// Device address of this device's scratch array, looked up once per device.
ce_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CE_ECUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return CE_ECUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return CE_OK;
}

}  // namespace

extern "C" {

ce_status ce_forward_noalloc(const void* logits, ce_dtype dt, ce_layout lg, int64_t N, int64_t V,
                             const void* targets, ce_index_dtype tdt, ce_layout tg,
                             float label_smoothing, int64_t ignore_index, float* loss, float* lse,
                             float* lse_lo, int32_t* argmax, void* cuda_stream) {
    if (N < 0 || V < 1 || (dt != CE_F32 && dt != CE_BF16 && dt != CE_F16)) return CE_EINVAL;
    const size_t need = N == 0 ? 0 : ce_workspace_size(N, V, dt, 0);
    if (need > kScratchBytes) return CE_EWORKSPACE;  // beyond the fixed array
    void* scratch = nullptr;
    if (need > 0) {
        const ce_status s = scratch_address(&scratch);
        if (s != CE_OK) return s;
    }
    // Every partial slot the merge reads is written by the same call first,
    // so nothing in the shared array has to start at zero.
    return ce_forward(logits, dt, lg, N, V, targets, tdt, tg, label_smoothing, ignore_index, loss,
                      lse, lse_lo, argmax, scratch, need > 0 ? kScratchBytes : 0, cuda_stream);
}

}  // extern "C"
