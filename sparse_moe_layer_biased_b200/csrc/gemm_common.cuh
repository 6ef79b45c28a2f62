// gemm_common.cuh — device helpers shared by the grouped-GEMM kernels (single-CTA and
// CTA-pair variants).
#pragma once

#include "sm100.cuh"

namespace moe {

// Clipped SwiGLU activation of one (gate, up) pair: min(silu(g), L) * clamp(u, -L, L),
// L = 0 meaning no clip ("MAX 中 Step-3.5-Flash 架构解析", sections
// "MoE共享专家、sigmoid 路由与激活裁剪" and "Step3p5Config配置项全解"). The comparisons keep a NaN.
// silu uses the fast exponential and division intrinsics: their error (a few fp32 ulp) is
// far below the bf16 rounding of h that follows.
__device__ __forceinline__ float swiglu_clip(float g, float u, float L)
{
    float a = __fdividef(g, 1.0f + __expf(-g));
    if (L > 0.0f) {
        a = a > L ? L : a;
        u = u > L ? L : (u < -L ? -L : u);
    }
    return a * u;
}

// Lane 0 waits, the whole warp learns the outcome (keeps warp-collective ops converged).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const WaitCfg &wc, volatile int *ab)
{
    bool ok = false;
    if ((threadIdx.x & 31) == 0)
        ok = mbar_wait(bar, parity, wc, ab);
    return __shfl_sync(0xFFFFFFFFu, ok, 0);
}

}  // namespace moe
