// noalloc.cu — moe_forward_noalloc: the whole layer for callers that cannot allocate
// device memory themselves.
//
// Who needs it: code that must not call the CUDA allocator when it runs, for example a
// serving runtime that hands almost all device memory to a fixed-size KV-cache pool at
// start-up (a later cudaMalloc then fails or fragments that pool), a decode loop with a
// latency budget where cudaMalloc / cudaFree may synchronise the device, or a plugin
// that runs inside a host framework without access to that framework's allocator.
// Those callers still own x, the weights and y; this entry point only removes the
// caller-provided workspace of moe_forward.
//
// How: the workspace lives in one file-scope device array of kScratchBytes (16 MiB).
// Under CUDA's default lazy module loading the array is created on a device by the first
// moe_forward_noalloc call there (the address lookup below loads this file's module);
// under eager loading it is created when the library's device code is loaded. Either way
// the device keeps it until the process exits. Host code cannot use the array's name as
// a device address (on the host it names a host-side stand-in), so every call looks up
// the device address with cudaGetSymbolAddress, with the caller's device current. The
// lookup is a runtime query that allocates nothing; doing it on every call means no
// saved address can outlive the context it belongs to (after cudaDeviceReset, or under
// another context bound to the same device, the module and its array may move).
#include "../../include/moe_b200.h"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the scratch array in the current context.
moe_status_t scratch_on_current_device(void **out)
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return MOE_ERR_CUDA;
    *out = p;
    return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_forward_noalloc(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wr,
                                            const float *bias, const uint16_t *W_gate_up, const uint16_t *W_down,
                                            const uint16_t *Wsh_gate_up, const uint16_t *Wsh_down, float *y,
                                            int32_t *topk_idx_out, float *topk_w_out, void *stream)
{
    size_t need = 0;
    moe_status_t st = moe_workspace_size(desc, &need);
    if (st != MOE_OK)
        return st;
    if (need > kScratchBytes)
        return MOE_ERR_WORKSPACE;  // this call needs more than the 16 MiB built-in scratch
    if (desc->T == 0)
        return MOE_OK;
    void *ws = nullptr;
    if ((st = scratch_on_current_device(&ws)) != MOE_OK)
        return st;
    // Every scratch byte that moe_forward reads is written earlier in the same call, so
    // nothing left over from the previous call needs clearing.
    return moe_forward(desc, x, Wr, bias, W_gate_up, W_down, Wsh_gate_up, Wsh_down, y, topk_idx_out, topk_w_out,
                       ws, kScratchBytes, stream);
}
