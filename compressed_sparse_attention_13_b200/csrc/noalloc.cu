// csa_decode_noalloc: csa_decode on a fixed device scratch area reserved
// statically in this file, for callers that cannot allocate device memory.
// Declared in include/csa.h, which lists the callers it serves and the
// rules for using it.
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = CSA_NOALLOC_SCRATCH_BYTES;

// One copy per CUDA context that loads this library, reserved when the
// module loads and freed only with the context.  Every call writes each byte
// before reading it, so the contents at load do not matter.
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the scratch area in the context current on the calling
// thread.  In host code the array's name is only a host-side stand-in, so the
// address is asked of the runtime.  It is asked on every call instead of
// being cached: a cached address would go stale after cudaDeviceReset (the
// module reloads into a new context) or when the caller makes another context
// current, and the lookup is a host-side table query once the module is
// loaded (it may load the module on the first call in a context).
int scratch_in_current_context(void** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return CSA_ERR_CUDA;
    *out = p;
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
    const int st = scratch_in_current_context(&scratch);
    if (st) return st;
    return csa_decode(p, batch, q, qI, qI_scales, w, kv, kv_scales, kI, kI_scales, max_blocks,
                      raw, n_raw, raw_pos0, q_pos, sinks, out, idx_out, scratch, kScratchBytes,
                      stream);
}
