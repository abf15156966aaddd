// csa_decode_noalloc: csa_decode on a fixed device scratch area reserved
// statically in this file, for callers that cannot allocate device memory.
// Declared in include/csa.h, which lists the callers it serves and the
// rules for using it.
#include <mutex>

#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = CSA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// One copy per device, reserved when the module loads; never freed.  Every
// call writes each byte before reading it, so the contents at load do not
// matter.
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_of[kMaxDevices] = {};

// Address of the scratch area on the current device, looked up once per
// device with that device current.
int scratch_on_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return CSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_of[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return CSA_ERR_CUDA;
        g_scratch_of[dev] = p;
    }
    *out = g_scratch_of[dev];
    return CSA_OK;
}

}  // namespace

extern "C" int csa_decode_noalloc(const csa_params* p, int32_t batch, const void* q,
                                  const void* qI, const void* qI_scales, const float* w,
                                  const void* kv, const void* kv_scales, const void* kI,
                                  const void* kI_scales, int64_t max_blocks, const void* raw,
                                  int64_t n_raw, const int64_t* raw_pos0, const int64_t* q_pos,
                                  const float* sinks, void* out, int32_t* idx_out,
                                  csa_stream_t stream) {
    if (!p || batch < 0 || max_blocks < 0) return CSA_ERR_ARG;
    if (batch == 0) return CSA_OK;
    // Reject a request larger than the scratch before touching the device.
    if (csa_workspace_size(p, CSA_OP_DECODE, batch, 1, max_blocks) > kScratchBytes)
        return CSA_ERR_WORKSPACE;
    void* scratch = nullptr;
    const int st = scratch_on_current_device(&scratch);
    if (st) return st;
    return csa_decode(p, batch, q, qI, qI_scales, w, kv, kv_scales, kI, kI_scales, max_blocks,
                      raw, n_raw, raw_pos0, q_pos, sinks, out, idx_out, scratch, kScratchBytes,
                      stream);
}
