// Status reporting for the vsa C ABI.
#include <cuda_runtime.h>

#include "vsa_internal.h"

extern "C" int vsa_check_status(vsa_plan_t plan, void* stream)
{
    if (!plan) return VSA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaStreamSynchronize(s) != cudaSuccess) return VSA_ERR_CUDA;
    unsigned int st = 0;
    if (cudaMemcpy(&st, plan->d_status, sizeof st, cudaMemcpyDeviceToHost) != cudaSuccess) return VSA_ERR_CUDA;
    if (st != 0 && cudaMemset(plan->d_status, 0, sizeof st) != cudaSuccess) return VSA_ERR_CUDA;
    if (st & VSA_DEV_TIMEOUT) return VSA_ERR_TIMEOUT;
    if (st & VSA_DEV_BADSTATE) return VSA_ERR_DEVICE;
    return VSA_OK;
}

extern "C" const char* vsa_status_string(int code)
{
    switch (code) {
    case VSA_OK: return "ok";
    case VSA_ERR_INVALID_ARG: return "invalid argument";
    case VSA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case VSA_ERR_ALIGNMENT: return "tensor pointer not 16-byte aligned";
    case VSA_ERR_CUDA: return "CUDA runtime or driver error";
    case VSA_ERR_OOM: return "device allocation failed";
    case VSA_ERR_TIMEOUT: return "device watchdog: a kernel wait expired";
    case VSA_ERR_DEVICE: return "device reported an inconsistent state";
    default: return "unknown status";
    }
}

extern "C" int vsa_version(void) { return VSA_VERSION; }
