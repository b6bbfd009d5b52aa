// Allocation-free variant of msa_fwd.
//
// msa_fwd needs a caller-provided device workspace (the block->query index,
// the fp32 output accumulators and the row sums).  Some callers cannot
// provide one: a plugin or custom-op host that owns every byte of device
// memory through its own pool and hands an operator only its inputs and
// outputs, or a latency-critical loop where a cudaMalloc/cudaFree (which
// can synchronise the whole device) is not allowed.  msa_fwd_noalloc serves
// them: its workspace is a fixed array in this library's device image, so
// the call itself allocates nothing.
//
// The array is kNoAllocScratchBytes (64 MiB).  Every GPU that loads this
// part of the library holds it until the process exits.  All calls on a
// device share it and it keeps the last call's contents; the forward path
// clears what must start at zero on every call.  Two calls whose work
// overlaps on the GPU (different streams, or different host threads) race
// on it: serialise them.
#include <mutex>

#include "../../include/msa.h"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)64 << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_fwd_scratch[kNoAllocScratchBytes];

std::mutex g_slot_mutex;
void* g_slot_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device, with that device current.  A failed look-up (the module
// holding the array could not be loaded, e.g. out of device memory) is not
// remembered: the next call tries again, and the runtime's error state is
// cleared so that it cannot surface in an unrelated later call.
int scratch_on_current_device(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MSA_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_slot_mutex);
    if (g_slot_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_fwd_scratch) != cudaSuccess || ptr == nullptr) {
            (void)cudaGetLastError();
            return MSA_ERR_LAUNCH;
        }
        g_slot_ptr[dev] = ptr;
    }
    *out = g_slot_ptr[dev];
    return MSA_OK;
}

}  // namespace
}  // namespace msa

extern "C" int msa_fwd_noalloc(const msa_dims* dims, const void* q, const void* k, const void* v,
                               const int32_t* idx, const int32_t* nsel, void* o, float* lse, void* stream)
{
    const size_t need = msa_workspace_size(dims, MSA_FWD);
    if (need == 0) return dims ? MSA_ERR_INVALID_DIMS : MSA_ERR_NULL_PTR;
    if (need > msa::kNoAllocScratchBytes) return MSA_ERR_WS_TOO_SMALL;
    void* ws = nullptr;
    const int rc = msa::scratch_on_current_device(&ws);
    if (rc != MSA_OK) return rc;
    return msa_fwd(dims, q, k, v, idx, nsel, o, lse, ws, msa::kNoAllocScratchBytes, stream);
}

extern "C" int msa_fwd_noalloc_status(void* stream, uint32_t* code)
{
    void* ws = nullptr;
    const int rc = msa::scratch_on_current_device(&ws);
    if (rc != MSA_OK) return rc == MSA_ERR_LAUNCH ? MSA_ERR_DEVICE : rc;
    return msa_check_status(ws, stream, code);
}
