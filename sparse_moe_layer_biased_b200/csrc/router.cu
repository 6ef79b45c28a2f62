// router.cu — fused router of the biased-sigmoid MoE layer on sm_100a.
//
// Layer step ("MAX 中 Step-3.5-Flash 架构解析", section "MoE共享专家、sigmoid 路由与激活裁剪"):
// scores = sigmoid(gate(x)) with the gate matmul in FP32, corrected = scores + router_bias
// used only to pick the top-k, weights taken from the uncorrected scores, normalised to
// sum 1 (norm_expert_weight) and multiplied by moe_router_scaling_factor; indices clamped
// to [0, E-1].
//
// A thread-block cluster of S CTAs owns a tile of TOK tokens (128, or 64 when E > 384) and
// all E experts; CTA s computes the fp32 logits of the tile over its K range
// [s*H/S, (s+1)*H/S) with tcgen05 MMAs (bf16 x bf16 products, fp32 accumulation in TMEM; two
// MMAs when E > 256) fed by a TMA ring, then parks the partial tile [TOK x E] in its shared
// memory (the idle ring). After a cluster barrier each CTA takes a share of the tile's tokens:
// one warp per token sums the S partials of each expert through distributed shared memory in
// rank order (a fixed order: the logits do not depend on timing), applies the sigmoid and the
// bias, and selects the top k by k+1 rounds of a warp-wide maximum over sortable 32-bit score
// keys (ties to the lower expert index: first within a lane, then across lanes by a second
// reduction that runs only when two lanes hold the maximum), which also gives the (k+1)-th for
// the margin. Lane l holds experts l, l + 32, ... (KPL of them, E <= 32 KPL). No logits reach
// global memory. S (1, 2, 4 or 8) is chosen so the grid covers the SMs about once.
#include "internal.h"

namespace moe {
namespace {

// warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 TMEM -> shared memory; all 16 warps select
// (the selection is latency-bound per warp: more warps per SM keep more tokens in flight)
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kTileM = 128;
constexpr int kBK = 64;                         // bf16 elements per 128-byte swizzled row
constexpr uint32_t kABytes = kTileM * kBK * 2;  // 16 KB
constexpr int kMaxStages = 8;

// Shared-memory layout for E_pad experts (a multiple of 16): a ring of stages (x tile +
// Wr rows of every expert), its barriers, and after the main loop the partial logits
// [tok][E_pad + 1] fp32 over the ring (row stride E_pad + 1 floats: conflict-free column
// writes from the TMEM epilogue).
struct Layout {
    uint32_t b_bytes, stage_bytes, bar_off, misc_off, total, tmem_cols, part_stride;
    int stages, tok;
    __host__ __device__ explicit Layout(int e_pad)
    {
        b_bytes = static_cast<uint32_t>(e_pad) * 128;
        stage_bytes = kABytes + b_bytes;
        const uint32_t fixed = 8 * (2 * kMaxStages + 2) + 64;
        int s = static_cast<int>((kMaxDynSmem - 1024 - fixed) / stage_bytes);
        stages = s > kMaxStages ? kMaxStages : s;
        part_stride = static_cast<uint32_t>(e_pad) + 1;
        const uint32_t ring = static_cast<uint32_t>(stages) * stage_bytes;
        tok = static_cast<uint32_t>(kTileM) * part_stride * 4 <= ring ? kTileM : kTileM / 2;
        bar_off = ring;
        misc_off = bar_off + 8 * (2 * kMaxStages + 2);
        total = misc_off + 16;
        uint32_t c = 32;
        while (c < static_cast<uint32_t>(e_pad))
            c <<= 1;
        tmem_cols = c;
    }
};

// Rank key of a biased score: larger key = ranked earlier. Order: value descending (-0 equal
// to +0), a NaN below every number; key 0 is an empty entry (an expert past E, or one already
// selected) and ranks below every real entry. A number's key is its order-preserving unsigned
// image plus one (at most 0xFF800001 for +inf), a NaN's key is 1.
__device__ __forceinline__ uint32_t rank_key(float b)
{
    if (b != b)
        return 1u;
    uint32_t u = (b == 0.0f) ? 0u : __float_as_uint(b);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return u + 1u;
}

__device__ __forceinline__ float key_value(uint32_t key)
{
    const uint32_t u = key - 1u;
    return __uint_as_float((u & 0x80000000u) ? (u ^ 0x80000000u) : ~u);
}

template <int KPL>
__global__ void __launch_bounds__(kThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wr,
                  const RouterArgs a, const int e_pad, const WaitCfg wc)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    const Layout L(e_pad);
    float *part = reinterpret_cast<float *>(smem);  // [tok][part_stride], over the ring after the main loop
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + kMaxStages;
    uint64_t *accf = empty + kMaxStages;
    uint64_t *drain = accf + 1;
    uint32_t *holder = reinterpret_cast<uint32_t *>(smem + L.misc_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc_off + 4);
    volatile int *ok_flag = reinterpret_cast<volatile int *>(smem + L.misc_off + 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = static_cast<int>(gridDim.x);  // the cluster: the S CTAs of one token tile
    const int rank = static_cast<int>(cluster_ctarank());
    const int m0 = static_cast<int>(blockIdx.y) * L.tok;
    const int nkb = a.H / (kBK * S);  // K stages of this CTA
    const int kb0 = rank * nkb;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        *ok_flag = 1;
        fence_barrier_init();
    }
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
            const uint32_t tx = kABytes + L.b_bytes;
            const int box = e_pad <= 256 ? e_pad : e_pad / 2;  // Wr rows per TMA box
            int issued = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % L.stages;
                if (!mbar_wait(&empty[s], ((kb / L.stages) & 1) ^ 1, wc, abort_flag))
                    break;
                mbar_arrive_expect_tx(&full[s], tx);
                uint8_t *A = smem + s * L.stage_bytes;
                uint8_t *B = A + kABytes;
                tma_load_2d(A, &tm_x, &full[s], (kb0 + kb) * kBK, m0);
                for (int r = 0; r < e_pad; r += box)
                    tma_load_2d(B + r * 128, &tm_wr, &full[s], (kb0 + kb) * kBK, r);
                ++issued;
            }
            for (int kb = issued > L.stages ? issued - L.stages : 0; kb < issued; ++kb)
                mbar_wait_drain(&full[kb % L.stages], (kb / L.stages) & 1, wc);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // N up to 256 per MMA: more than 256 experts take two MMAs
            const int n0 = e_pad < 256 ? e_pad : 256;
            const int n1 = e_pad - n0;
            const uint32_t id0 = idesc_bf16_f32(kTileM, n0);
            const uint32_t id1 = idesc_bf16_f32(kTileM, n1 > 0 ? n1 : 16);
            bool ok = true;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % L.stages;
                if (!mbar_wait(&full[s], (kb / L.stages) & 1, wc, abort_flag)) {
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
    } else if (warp < 6) {
        // warps 2-5: TMEM lane quarter q (token rows 32q .. 32q+31) -> the partial tile. Every
        // MMA has completed (accf), so every stage of the ring has been consumed.
        bool ok = false;
        if (lane == 0)
            ok = mbar_wait(accf, 0, wc, abort_flag);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        tc_fence_after();
        if (ok) {
            const int q = warp & 3;
            const int row = q * 32 + lane;
            const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16);
            for (int c0 = 0; c0 < e_pad; c0 += 32) {
                float v[32];
                tmem_load32(tbase + c0, v);
                if (row < L.tok) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (c0 + i < e_pad)
                            part[row * L.part_stride + c0 + i] = v[i];
                }
            }
        } else if (lane == 0) {
            *ok_flag = 0;
        }
    }

    // The partial tiles of all S CTAs are complete and visible cluster-wide.
    tc_fence_before();
    cluster_sync_all();

    bool all_ok = true;
    for (int p = 0; p < S; ++p)
        all_ok = all_ok && dsmem_ld_s32(dsmem_addr(smem_u32(const_cast<int *>(ok_flag)), p)) != 0;
    if (all_ok) {
        // this CTA's share of the tile's tokens, one warp per token
        const int per = (L.tok + S - 1) / S;
        const int t_hi = (rank + 1) * per < L.tok ? (rank + 1) * per : L.tok;
        const float *peer[8];
#pragma unroll
        for (int p = 0; p < 8; ++p)
            peer[p] = peer_ptr(part, static_cast<uint32_t>(p < S ? p : 0));
        const int rounds = a.k < a.E ? a.k + 1 : a.k;
        // this lane's experts' biases, the same for every token
        float bias_r[KPL];
#pragma unroll
        for (int i = 0; i < KPL; ++i)
            bias_r[i] = lane + 32 * i < a.E ? a.bias[lane + 32 * i] : 0.0f;
        for (int tt = rank * per + warp; tt < t_hi; tt += kWarps) {
            const int t = m0 + tt;
            if (t >= a.T)
                break;
            // lane l holds experts l, l + 32, ...: logit = sum of the S partials in rank order
            uint32_t key[KPL];
            float sc[KPL];
#pragma unroll
            for (int i = 0; i < KPL; ++i) {
                const int e = lane + 32 * i;
                key[i] = 0u;
                sc[i] = 0.0f;
                if (e < a.E) {
                    const int off = tt * static_cast<int>(L.part_stride) + e;
                    float l = 0.0f;
#pragma unroll
                    for (int p = 0; p < 8; ++p)
                        if (p < S)
                            l += peer[p][off];
                    const float s = 1.0f / (1.0f + expf(-l));
                    key[i] = rank_key(s + bias_r[i]);
                    sc[i] = s;
                }
            }
            // k (+1 for the margin) rounds of a warp-wide maximum: lane j keeps round j's
            // expert and score; the normalisation sum and the margin keys are warp-uniform,
            // accumulated in rank order
            const int k = a.k;
            int my_e = 0;
            uint32_t key_k = 0u, key_k1 = 0u;
            float my_s = 0.0f, sum = 0.0f;
            for (int j = 0; j < rounds; ++j) {
                // this lane's best entry: highest key, lowest index among equal keys
                uint32_t best = 0u;
                int bi = 0;
#pragma unroll
                for (int i = 0; i < KPL; ++i) {
                    const bool gt = key[i] > best;
                    best = gt ? key[i] : best;
                    bi = gt ? i : bi;
                }
                const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, best);
                const unsigned holders = __ballot_sync(0xFFFFFFFFu, best == m && m != 0u);
                int win = holders ? __ffs(holders) - 1 : 0;
                if (__popc(holders) > 1) {
                    // equal keys in several lanes: the lowest expert index wins
                    const uint32_t ex = (holders >> lane) & 1u ? static_cast<uint32_t>(lane + 32 * bi) : 0xFFFFFFFFu;
                    const uint32_t emin = __reduce_min_sync(0xFFFFFFFFu, ex);
                    win = static_cast<int>(emin & 31u);
                }
                const int we = __shfl_sync(0xFFFFFFFFu, lane + 32 * bi, win);
                float ws = 0.0f;
#pragma unroll
                for (int i = 0; i < KPL; ++i)
                    ws = i == bi ? sc[i] : ws;
                ws = __shfl_sync(0xFFFFFFFFu, ws, win);
                ws = m != 0u ? ws : 0.0f;  // no entry left (cannot happen with k + 1 <= E rounds)
                if (lane == win && m != 0u) {
#pragma unroll
                    for (int i = 0; i < KPL; ++i)
                        key[i] = i == bi ? 0u : key[i];
                }
                if (lane == (j & 31) && j < k) {
                    my_e = we;
                    my_s = ws;
                }
                if (j < k)
                    sum += ws;
                key_k = j + 1 == k ? m : key_k;
                key_k1 = j == k ? m : key_k1;
            }
            if (lane < k) {
                int e = my_e;
                e = e < 0 ? 0 : (e > a.E - 1 ? a.E - 1 : e);
                float w;
                if (a.norm)
                    w = sum > 0.0f ? a.scale * (my_s / sum) : a.scale / static_cast<float>(k);
                else
                    w = a.scale * my_s;
                a.idx[static_cast<int64_t>(t) * k + lane] = e;
                a.w[static_cast<int64_t>(t) * k + lane] = w;
            }
            if (lane == 0 && a.margin)
                a.margin[t] = k < a.E ? key_value(key_k) - key_value(key_k1) : __int_as_float(0x7F800000);
        }
    }

    // Peers have finished reading this CTA's partial tile before any CTA exits.
    cluster_sync_all();

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L.tmem_cols);
    }
}

cudaError_t launch_impl(const CUtensorMap &tm_x, const CUtensorMap &tm_wr, const RouterArgs &a,
                        const WaitCfg &wc, cudaStream_t stream)
{
    const RouterSplit sp = router_split(a.E, a.T, a.H, a.num_sms);
    const Layout L(sp.e_pad);
    const int smem = static_cast<int>(L.total) + 1024;
    // keys per lane: the smallest of 4, 8, 12, 16 covering E_pad experts over 32 lanes
    const int kpl = (sp.e_pad + 31) / 32;
    auto kernel = kpl <= 4 ? router_kernel<4> : (kpl <= 8 ? router_kernel<8> : (kpl <= 12 ? router_kernel<12> : router_kernel<16>));
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sp.ks, (a.T + L.tok - 1) / L.tok, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = sp.ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kernel, tm_x, tm_wr, a, sp.e_pad, wc);
    if (err != cudaSuccess)
        return err;
    return cudaGetLastError();
}

}  // namespace

// K split S (a power of two up to 8 that divides H / 64) so that about one CTA runs per SM:
// token tiles x S ~ num_sms. All experts in every CTA (E padded to a multiple of 16; above
// 256 experts the Wr rows of a stage come as two boxes of E_pad / 2 rows).
RouterSplit router_split(int E, int T, int H, int num_sms)
{
    const int e_pad = (E + 15) / 16 * 16;
    const Layout L(e_pad);
    const int tiles = (T + L.tok - 1) / L.tok;
    int ks = 1;
    while (ks < 8 && tiles * ks * 2 <= num_sms && (H / kBK) % (ks * 2) == 0)
        ks *= 2;
    RouterSplit r;
    r.e_pad = e_pad;
    r.ks = ks;
    r.box_rows = e_pad <= 256 ? e_pad : e_pad / 2;
    return r;
}

cudaError_t launch_router(const CUtensorMap &tm_x, const CUtensorMap &tm_wr, const RouterArgs &a,
                          const WaitCfg &wc, cudaStream_t stream)
{
    return launch_impl(tm_x, tm_wr, a, wc, stream);
}

}  // namespace moe
