// qsa_decode_step_noalloc: the decode step for callers that cannot allocate
// device memory at all, not even a workspace.
//
// Some callers can't call cudaMalloc: serving engines that carve all device
// memory into their own pool up front and forbid allocations outside it,
// plugin hosts that hand a plugin a stream and tensors but no allocator or
// workspace, and latency-critical loops that cannot afford the implicit
// device-wide synchronisation cudaMalloc/cudaFree may cause. For them this
// entry point takes its scratch from a fixed array in the library's own device
// memory (reserved by the driver when the library's device code is loaded on a
// GPU, and held until the process exits) instead of a caller workspace.
#include <cuda_runtime.h>

#include "../../include/qsa.h"
#include "kernels.h"

namespace {

// Scratch of qsa_decode_step_noalloc. 16 MiB covers the decode workspace of,
// e.g., 8 sequences of 256K cached tokens or 1 sequence of 4M.
constexpr size_t kScratchBytes = (size_t)QSA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

// Device address of g_decode_scratch in the current context. In host code the
// array's name is only a host-side stand-in; its device address comes from
// cudaGetSymbolAddress, asked on every call: the address belongs to the
// context that loaded the library's device code, and a context that is
// destroyed and created again (cudaDeviceReset) may load it elsewhere. The
// first call in a context loads that code, so it must not fall inside a
// stream capture.
cudaError_t scratch_ptr(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" qsa_status qsa_decode_step_noalloc(const qsa_config* cfg, int32_t batch,
                                              const int64_t* pos, const qsa_bf16* q,
                                              const qsa_bf16* k, const qsa_bf16* v,
                                              const qsa_bf16* idx_q, const qsa_bf16* idx_k,
                                              qsa_bf16* k_cache, qsa_bf16* v_cache,
                                              qsa_bf16* idx_k_cache, qsa_bf16* pooled,
                                              int64_t cap, const float* rms_w, qsa_bf16* out,
                                              int32_t* sel_out, int32_t* nsel_out,
                                              qsa_stream stream) {
    size_t need = 0;
    qsa_status st = qsa_workspace_size(cfg, QSA_OP_DECODE_STEP, batch, cap, 0, &need);
    if (st != QSA_OK) return st;
    if (need > kScratchBytes)
        return (qsa_status)qsa::report_error(
            QSA_ERR_WORKSPACE,
            "qsa_decode_step_noalloc: batch=%d, cap=%lld needs %zu bytes of decode scratch, above "
            "its fixed %zu bytes; use qsa_decode_step with a workspace",
            batch, (long long)cap, need, kScratchBytes);
    void* ws = nullptr;
    cudaError_t e = scratch_ptr(&ws);
    if (e != cudaSuccess)
        return (qsa_status)qsa::report_error(QSA_ERR_CUDA, "qsa_decode_step_noalloc set-up: %s",
                                             cudaGetErrorString(e));
    // The status header and the selection state must start at zero; the array
    // may hold another batch size's layout from an earlier call. The step
    // checks every argument before it clears them and launches.
    return (qsa_status)qsa::decode_step_cleared(cfg, batch, pos, q, k, v, idx_q, idx_k, k_cache, v_cache,
                                                idx_k_cache, pooled, cap, rms_w, out, sel_out, nsel_out, ws,
                                                kScratchBytes, stream);
}
