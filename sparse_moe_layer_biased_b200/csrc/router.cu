// router.cu — fused router of the biased-sigmoid MoE layer on sm_100a.
//
// Layer step ("MAX 中 Step-3.5-Flash 架构解析", section "MoE共享专家、sigmoid 路由与激活裁剪"):
// scores = sigmoid(gate(x)) with the gate matmul in FP32, corrected = scores + router_bias
// used only to pick the top-k, weights taken from the uncorrected scores, normalised to
// sum 1 (norm_expert_weight) and multiplied by moe_router_scaling_factor; indices clamped
// to [0, E-1].
//
// One CTA owns 128 tokens. The logits tile [128 tokens x E] is one tcgen05 GEMM
// (bf16 x bf16 products, fp32 accumulation in TMEM; E up to 512 columns as two MMAs of
// N <= 256). TMA streams x and Wr K-slices through a 2-4 stage mbarrier ring. The
// epilogue gives each TMEM lane (= token) to one thread, which reads its E logits in
// 32-column chunks and keeps a sorted top-(k+1) list in registers: no logits reach HBM.
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue
constexpr int kTileM = 128;
constexpr int kBK = 64;                          // bf16 elements per 128-byte swizzled row
constexpr uint32_t kABytes = kTileM * kBK * 2;   // 16 KB
constexpr int kBRows = 16;                       // rows per Wr TMA box

struct Layout {
    int e_pad, n0, n1, stages;
    uint32_t b_bytes, stage_bytes, bias_off, bar_off, misc_off, total;
    uint32_t tmem_cols;
};

__host__ __device__ inline Layout make_layout(int E)
{
    Layout L{};
    L.e_pad = (E + 15) / 16 * 16;
    L.n0 = L.e_pad < 256 ? L.e_pad : 256;
    L.n1 = L.e_pad - L.n0;
    L.b_bytes = (static_cast<uint32_t>(L.e_pad) * 128 + 1023) / 1024 * 1024;
    L.stage_bytes = kABytes + L.b_bytes;
    const uint32_t budget = kMaxDynSmem - 1024 - 4096;
    int s = static_cast<int>(budget / L.stage_bytes);
    L.stages = s > 4 ? 4 : s;
    L.bias_off = L.stages * L.stage_bytes;
    L.bar_off = L.bias_off + (static_cast<uint32_t>(L.e_pad) * 4 + 15) / 16 * 16;
    L.misc_off = L.bar_off + 8 * (2 * 4 + 2);
    L.total = L.misc_off + 16;
    uint32_t c = 32;
    while (c < static_cast<uint32_t>(L.e_pad))
        c <<= 1;
    L.tmem_cols = c;
    return L;
}

// Rank key of a biased score: larger key = ranked earlier. Order: value descending
// (-0 equal to +0), a NaN below every number, ties to the lower expert index.
__device__ __forceinline__ uint64_t rank_key(float b, int e)
{
    uint32_t u;
    if (b != b) {
        u = 0u;
    } else {
        u = (b == 0.0f) ? 0u : __float_as_uint(b);
        u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    }
    return (static_cast<uint64_t>(u) << 32) | static_cast<uint32_t>(0xFFFFFFFFu - static_cast<uint32_t>(e));
}

__device__ __forceinline__ float key_value(uint64_t key)
{
    const uint32_t u = static_cast<uint32_t>(key >> 32);
    return __uint_as_float((u & 0x80000000u) ? (u ^ 0x80000000u) : ~u);
}

__device__ __forceinline__ int key_expert(uint64_t key)
{
    return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(key));
}

template <int KMAX>
__global__ void __launch_bounds__(kThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wr,
                  const RouterArgs a, const WaitCfg wc)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    const Layout L = make_layout(a.E);
    float *bias_s = reinterpret_cast<float *>(smem + L.bias_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + 4;
    uint64_t *accf = empty + 4;
    uint64_t *drain = accf + 1;
    uint32_t *holder = reinterpret_cast<uint32_t *>(smem + L.misc_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc_off + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kTileM;
    const int nkb = a.H / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 4; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    for (int e = threadIdx.x; e < L.e_pad; e += kThreads)
        bias_s[e] = e < a.E ? a.bias[e] : 0.0f;
    if (warp == 1) {
        tmem_alloc(holder, L.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *holder;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_map(&tm_x);
            tma_prefetch_map(&tm_wr);
            const uint32_t tx = kABytes + static_cast<uint32_t>(L.e_pad) * 128;
            int issued = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % L.stages;
                const uint32_t ph = (kb / L.stages) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, wc, abort_flag))
                    break;
                mbar_arrive_expect_tx(&full[s], tx);
                uint8_t *A = smem + s * L.stage_bytes;
                uint8_t *B = A + kABytes;
                tma_load_2d(A, &tm_x, &full[s], kb * kBK, m0);
                for (int r = 0; r < L.e_pad; r += kBRows)
                    tma_load_2d(B + r * 128, &tm_wr, &full[s], kb * kBK, r);
                ++issued;
            }
            for (int kb = issued > L.stages ? issued - L.stages : 0; kb < issued; ++kb)
                mbar_wait_drain(&full[kb % L.stages], (kb / L.stages) & 1, wc);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id0 = idesc_bf16_f32(kTileM, L.n0);
            const uint32_t id1 = idesc_bf16_f32(kTileM, L.n1 > 0 ? L.n1 : 16);
            bool ok = true;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % L.stages;
                const uint32_t ph = (kb / L.stages) & 1;
                if (!mbar_wait(&full[s], ph, wc, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + s * L.stage_bytes);
                const uint32_t b_addr = a_addr + kABytes;
                const uint64_t ad = sdesc_kmajor_sw128(a_addr);
                const uint64_t bd0 = sdesc_kmajor_sw128(b_addr);
                const uint64_t bd1 = sdesc_kmajor_sw128(b_addr + static_cast<uint32_t>(L.n0) * 128);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    const uint32_t acc = (kb | kk) != 0;
                    umma_bf16(tmem, ad + 2 * kk, bd0 + 2 * kk, id0, acc);
                    if (L.n1 > 0)
                        umma_bf16(tmem + L.n0, ad + 2 * kk, bd1 + 2 * kk, id1, acc);
                }
                umma_commit(&empty[s]);
            }
            if (ok)
                umma_commit(accf);
            umma_commit(drain);
            mbar_wait_drain(drain, 0, wc);
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const int t = m0 + row;
        bool ok = false;
        if (lane == 0)
            ok = mbar_wait(accf, 0, wc, abort_flag);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        tc_fence_after();
        if (ok) {
            uint64_t keys[KMAX + 1];
            float sv[KMAX + 1];
#pragma unroll
            for (int j = 0; j <= KMAX; ++j) {
                keys[j] = 0;
                sv[j] = 0.0f;
            }
            const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16);
            for (int c0 = 0; c0 < a.E; c0 += 32) {
                float v[32];
                tmem_load32(tbase + c0, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int e = c0 + i;
                    if (e < a.E) {
                        const float s = 1.0f / (1.0f + expf(-v[i]));
                        const float b = s + bias_s[e];
                        const uint64_t key = rank_key(b, e);
                        if (key > keys[KMAX]) {
                            keys[KMAX] = key;
                            sv[KMAX] = s;
#pragma unroll
                            for (int j = KMAX; j > 0; --j) {
                                if (keys[j] > keys[j - 1]) {
                                    const uint64_t tk = keys[j];
                                    keys[j] = keys[j - 1];
                                    keys[j - 1] = tk;
                                    const float ts = sv[j];
                                    sv[j] = sv[j - 1];
                                    sv[j - 1] = ts;
                                }
                            }
                        }
                    }
                }
            }
            if (t < a.T) {
                const int k = a.k;
                float sum = 0.0f;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (j < k)
                        sum += sv[j];
                float bk = 0.0f, bk1 = 0.0f;
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (j < k) {
                        int e = key_expert(keys[j]);
                        e = e < 0 ? 0 : (e > a.E - 1 ? a.E - 1 : e);
                        float w;
                        if (a.norm)
                            w = sum > 0.0f ? a.scale * (sv[j] / sum) : a.scale / static_cast<float>(k);
                        else
                            w = a.scale * sv[j];
                        a.idx[static_cast<int64_t>(t) * k + j] = e;
                        a.w[static_cast<int64_t>(t) * k + j] = w;
                    }

                }
                // k-th and (k+1)-th keys picked by a compare-and-select chain (a dynamic
                // index would move the list to local memory)
                uint64_t key_k = 0, key_k1 = 0;
#pragma unroll
                for (int j = 0; j <= KMAX; ++j) {
                    const bool at_k = (j + 1 == k), at_k1 = (j == k);
                    key_k = at_k ? keys[j] : key_k;
                    key_k1 = at_k1 ? keys[j] : key_k1;
                    asm volatile("" : "+l"(key_k), "+l"(key_k1));
                }
                bk = key_value(key_k);
                bk1 = key_value(key_k1);
                if (a.margin)
                    a.margin[t] = k < a.E ? bk - bk1 : __int_as_float(0x7F800000);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L.tmem_cols);
    }
}

template <int KMAX>
cudaError_t launch_impl(const CUtensorMap &tm_x, const CUtensorMap &tm_wr, const RouterArgs &a,
                        const WaitCfg &wc, cudaStream_t stream)
{
    const Layout L = make_layout(a.E);
    const int smem = static_cast<int>(L.total) + 1024;
    cudaError_t err = cudaFuncSetAttribute(router_kernel<KMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    const int grid = (a.T + kTileM - 1) / kTileM;
    router_kernel<KMAX><<<grid, kThreads, smem, stream>>>(tm_x, tm_wr, a, wc);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const CUtensorMap &tm_x, const CUtensorMap &tm_wr, const RouterArgs &a,
                          const WaitCfg &wc, cudaStream_t stream)
{
    if (a.k <= 4)
        return launch_impl<4>(tm_x, tm_wr, a, wc, stream);
    if (a.k <= 8)
        return launch_impl<8>(tm_x, tm_wr, a, wc, stream);
    if (a.k <= 16)
        return launch_impl<16>(tm_x, tm_wr, a, wc, stream);
    return launch_impl<32>(tm_x, tm_wr, a, wc, stream);
}

}  // namespace moe
