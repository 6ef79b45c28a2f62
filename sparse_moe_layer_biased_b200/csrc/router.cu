// router.cu — fused router of the biased-sigmoid MoE layer on sm_100a.
//
// Layer step ("MAX 中 Step-3.5-Flash 架构解析", section "MoE共享专家、sigmoid 路由与激活裁剪"):
// scores = sigmoid(gate(x)) with the gate matmul in FP32, corrected = scores + router_bias
// used only to pick the top-k, weights taken from the uncorrected scores, normalised to
// sum 1 (norm_expert_weight) and multiplied by moe_router_scaling_factor; indices clamped
// to [0, E-1].
//
// A thread-block cluster of NS CTAs owns 128 tokens; CTA r owns the experts of slice r
// (SL experts, a multiple of 16, up to 512). Each CTA computes its logits tile
// [128 tokens x SL] with tcgen05 MMAs (bf16 x bf16 products, fp32 accumulation in TMEM;
// two MMAs when SL > 256) fed by a TMA ring,
// then gives each TMEM lane (= token) to one thread, which keeps a sorted top-(k+1) list
// of its slice in registers. The lists meet in CTA 0 through distributed shared memory,
// where each thread merges the NS lists of its token and writes ids, weights and margin.
// No logits reach global memory. NS is chosen so the grid covers the SMs about once:
// decode-sized calls split the experts over up to 8 CTAs, large calls use NS = 1.
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue
constexpr int kTileM = 128;
constexpr int kBK = 64;                         // bf16 elements per 128-byte swizzled row
constexpr uint32_t kABytes = kTileM * kBK * 2;  // 16 KB
constexpr int kMaxStages = 8;

template <int KMAX>
struct Layout {
    uint32_t b_bytes, stage_bytes, list_off, bias_off, bar_off, misc_off, total, tmem_cols;
    int stages;
    __host__ __device__ explicit Layout(int sl)
    {
        b_bytes = (static_cast<uint32_t>(sl) * 128 + 1023) / 1024 * 1024;
        stage_bytes = kABytes + b_bytes;
        const uint32_t list_bytes = kTileM * (KMAX + 1) * 12;
        const uint32_t fixed = list_bytes + static_cast<uint32_t>(sl) * 4 + 8 * (2 * kMaxStages + 2) + 64;
        int s = static_cast<int>((kMaxDynSmem - 1024 - fixed) / stage_bytes);
        stages = s > kMaxStages ? kMaxStages : s;
        list_off = stages * stage_bytes;  // keys [128][KMAX+1] u64, then scores [128][KMAX+1] f32
        bias_off = list_off + list_bytes;
        bar_off = (bias_off + static_cast<uint32_t>(sl) * 4 + 7) / 8 * 8;
        misc_off = bar_off + 8 * (2 * kMaxStages + 2);
        total = misc_off + 16;
        uint32_t c = 32;
        while (c < static_cast<uint32_t>(sl))
            c <<= 1;
        tmem_cols = c;
    }
};

// Rank key of a biased score: larger key = ranked earlier. Order: value descending
// (-0 equal to +0), a NaN below every number, ties to the lower expert index. Key 0
// (an empty list entry) ranks below every real entry.
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

// Insert (key, s) into the descending register list keys[0..KMAX] (fully unrolled).
template <int KMAX>
__device__ __forceinline__ void list_insert(uint64_t (&keys)[KMAX + 1], float (&sv)[KMAX + 1], uint64_t key, float s)
{
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

template <int KMAX>
__global__ void __launch_bounds__(kThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wr,
                  const RouterArgs a, const int sl, const WaitCfg wc)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    const Layout<KMAX> L(sl);
    uint64_t *list_keys = reinterpret_cast<uint64_t *>(smem + L.list_off);
    float *list_s = reinterpret_cast<float *>(smem + L.list_off + kTileM * (KMAX + 1) * 8);
    float *bias_s = reinterpret_cast<float *>(smem + L.bias_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + kMaxStages;
    uint64_t *accf = empty + kMaxStages;
    uint64_t *drain = accf + 1;
    uint32_t *holder = reinterpret_cast<uint32_t *>(smem + L.misc_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc_off + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int ns = static_cast<int>(gridDim.x);
    const int e0 = static_cast<int>(blockIdx.x) * sl;
    const int ne = (a.E - e0) < sl ? (a.E - e0) : sl;  // experts of this slice (>= 1)
    const int m0 = blockIdx.y * kTileM;
    const int nkb = a.H / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    for (int e = threadIdx.x; e < sl; e += kThreads)
        bias_s[e] = e < ne ? a.bias[e0 + e] : 0.0f;
    if (warp == 1) {
        tmem_alloc(holder, L.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *holder;
    const int box = sl <= 256 ? sl : sl / 2;  // Wr rows per TMA box (one or two per stage)

    // registers of the epilogue thread's list (kept across the cluster barrier in CTA 0)
    uint64_t keys[KMAX + 1];
    float sv[KMAX + 1];
#pragma unroll
    for (int j = 0; j <= KMAX; ++j) {
        keys[j] = 0;
        sv[j] = 0.0f;
    }
    const int q = warp & 3;
    const int row = q * 32 + lane;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_map(&tm_x);
            tma_prefetch_map(&tm_wr);
            const uint32_t tx = kABytes + static_cast<uint32_t>(sl) * 128;
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
                for (int r = 0; r < sl; r += box)
                    tma_load_2d(B + r * 128, &tm_wr, &full[s], kb * kBK, e0 + r);
                ++issued;
            }
            for (int kb = issued > L.stages ? issued - L.stages : 0; kb < issued; ++kb)
                mbar_wait_drain(&full[kb % L.stages], (kb / L.stages) & 1, wc);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // N up to 256 per MMA: a slice of more than 256 experts takes two MMAs
            const int n0 = sl < 256 ? sl : 256;
            const int n1 = sl - n0;
            const uint32_t id0 = idesc_bf16_f32(kTileM, n0);
            const uint32_t id1 = idesc_bf16_f32(kTileM, n1 > 0 ? n1 : 16);
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
                const uint64_t ad = sdesc_kmajor_sw128(a_addr);
                const uint64_t bd0 = sdesc_kmajor_sw128(a_addr + kABytes);
                const uint64_t bd1 = sdesc_kmajor_sw128(a_addr + kABytes + static_cast<uint32_t>(n0) * 128);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    umma_bf16(tmem, ad + 2 * kk, bd0 + 2 * kk, id0, (kb | kk) != 0);
                    if (n1 > 0)
                        umma_bf16(tmem + n0, ad + 2 * kk, bd1 + 2 * kk, id1, (kb | kk) != 0);
                }
                umma_commit(&empty[s]);
            }
            if (ok)
                umma_commit(accf);
            umma_commit(drain);
            mbar_wait_drain(drain, 0, wc);
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31; one thread per token row
        bool ok = false;
        if (lane == 0)
            ok = mbar_wait(accf, 0, wc, abort_flag);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        tc_fence_after();
        if (ok) {
            const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16);
            for (int c0 = 0; c0 < ne; c0 += 32) {
                float v[32];
                tmem_load32(tbase + c0, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int e = c0 + i;
                    if (e < ne) {
                        const float s = 1.0f / (1.0f + expf(-v[i]));
                        const float b = s + bias_s[e];
                        list_insert<KMAX>(keys, sv, rank_key(b, e0 + e), s);
                    }
                }
            }
        }
        if (rank != 0) {
#pragma unroll
            for (int j = 0; j <= KMAX; ++j) {
                list_keys[row * (KMAX + 1) + j] = keys[j];
                list_s[row * (KMAX + 1) + j] = sv[j];
            }
        }
    }

    // Lists of CTAs 1..ns-1 become visible to CTA 0; every thread of every CTA gets here.
    cluster_sync_all();

    if (rank == 0 && warp >= 2) {
        const uint32_t keys_local = smem_u32(list_keys + row * (KMAX + 1));
        const uint32_t s_local = smem_u32(list_s + row * (KMAX + 1));
        for (int p = 1; p < ns; ++p) {
            const uint32_t kp = dsmem_addr(keys_local, p);
            const uint32_t sp = dsmem_addr(s_local, p);
            for (int j = 0; j <= KMAX; ++j) {
                const uint64_t key = dsmem_ld_u64(kp + 8 * j);
                if (key <= keys[KMAX])
                    break;  // peer lists are sorted: nothing further can enter
                list_insert<KMAX>(keys, sv, key, dsmem_ld_f32(sp + 4 * j));
            }
        }
        const int t = m0 + row;
        if (t < a.T) {
            const int k = a.k;
            float sum = 0.0f;
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                if (j < k)
                    sum += sv[j];
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
            if (a.margin)
                a.margin[t] = k < a.E ? key_value(key_k) - key_value(key_k1) : __int_as_float(0x7F800000);
        }
    }

    // CTA 0 has finished reading its peers' shared memory before any CTA exits.
    cluster_sync_all();

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
    const RouterSplit sp = router_split(a.E, a.T, a.num_sms);
    const Layout<KMAX> L(sp.sl);
    const int smem = static_cast<int>(L.total) + 1024;
    cudaError_t err = cudaFuncSetAttribute(router_kernel<KMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sp.ns, (a.T + kTileM - 1) / kTileM, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = sp.ns;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, router_kernel<KMAX>, tm_x, tm_wr, a, sp.sl, wc);
    if (err != cudaSuccess)
        return err;
    return cudaGetLastError();
}

}  // namespace

// Enough CTAs to cover the SMs once: with few token tiles (decode) the experts are split
// over up to 8 CTAs; with many token tiles each CTA keeps all experts, so x is read once.
// Slices above 256 experts are a multiple of 32, loaded as two Wr boxes of sl / 2 rows.
RouterSplit router_split(int E, int T, int num_sms)
{
    const int tiles = (T + kTileM - 1) / kTileM;
    const int e_pad = (E + 15) / 16 * 16;
    int ns = num_sms / tiles;
    ns = ns < 1 ? 1 : (ns > 8 ? 8 : ns);
    ns = ns > e_pad / 16 ? e_pad / 16 : ns;
    int sl = ((e_pad + ns - 1) / ns + 15) / 16 * 16;
    if (sl > 256)
        sl = (sl + 31) / 32 * 32;
    RouterSplit r;
    r.sl = sl;
    r.ns = (E + sl - 1) / sl;
    r.box_rows = sl <= 256 ? sl : sl / 2;
    return r;
}

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
