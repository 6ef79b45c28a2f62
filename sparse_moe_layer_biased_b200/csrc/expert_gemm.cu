// expert_gemm.cu — grouped expert GEMMs of the MoE layer on sm_100a (tcgen05 + TMEM + TMA).
//
// Layer step ("MAX 中 Step-3.5-Flash 架构解析", section "MoE共享专家、sigmoid 路由与激活裁剪"):
// output = routed_moe(x) + shared_expert(x); each expert is a SwiGLU MLP whose gated
// activation is built from the concatenated gate/up projection with a per-layer clip
// limit (swiglu_limits / swiglu_limits_shared, 0 = no clip, section
// "Step3p5Config配置项全解"). The fused [2I, H] gate_up and [H, I] down layouts follow
// the 24 MiB / 12 MiB BF16 expert tensors of the miles Step-5-Preview page, section 5.3.
//
// Both kernels are "swap-AB": expert weight rows fill the 128-lane M side of the UMMA
// and the tokens of one expert chunk (up to BN rows, rounded up to a multiple of 16) are
// the N side, so a ragged group wastes at most 15 token columns and a decode-sized group
// of one or two tokens still streams full weight tiles. A stage holds MT weight tiles of
// 128 rows that share one token tile: MT = 2 halves how often a token chunk is re-read
// from L2 per weight byte (the token tile is reused by two MMAs per K step).
//
// Roles per CTA (persistent, one CTA per SM, static round-robin over tiles):
//   warp 0      TMA producer: per 64-wide K slice, one box with the MT weight tiles and
//               one box of BN token rows
//   warp 1      MMA issuer (one thread) and TMEM owner; 2 buffers x MT accumulators x BN
//               fp32 columns, so the epilogue of one tile overlaps the mainloop of the next
//   warps 2..5  epilogue: TMEM -> registers -> activation / weighting -> global
// Every wait is bounded (mbar_wait); on expiry the CTA drains its own copies and MMAs,
// frees TMEM and returns with the device error word set.
#include "epilogue.cuh"

namespace moe {
namespace {

constexpr int kThreads = 192;
constexpr int kBK = 64;
constexpr uint32_t kATileBytes = 128 * 128;  // 128 weight rows x 64 bf16

// Ring geometry: token chunks of at most BN rows, S stages, MT weight tiles per stage.
template <int BN, int S, int MT>
struct Geo {
    static constexpr uint32_t kABytes = MT * kATileBytes;
    static constexpr uint32_t kBBytes = BN * 128;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr uint32_t kBarOff = S * kStageBytes;
    static constexpr uint32_t kMiscOff = kBarOff + 8 * (2 * S + 5);
    static constexpr uint32_t kSmemBytes = kMiscOff + 16 + 1024;
    static constexpr uint32_t kBufCols = MT * BN;  // one TMEM buffer: MT accumulators of BN columns
    static constexpr uint32_t kTmemCols = 2 * kBufCols < 32 ? 32 : 2 * kBufCols;
    static_assert(kStageBytes % 1024 == 0, "stages must stay 1024-byte aligned");
    static_assert(kSmemBytes <= kMaxDynSmem, "ring exceeds shared memory");
    static_assert((kTmemCols & (kTmemCols - 1)) == 0 && kTmemCols <= 512, "TMEM allocation");
};

struct Ring {
    uint64_t *full, *empty, *accf, *acce, *drain;
    uint32_t *holder;
    volatile int *abort_flag;
};

template <class G, int S>
__device__ __forceinline__ uint8_t *ring_setup(uint8_t *smem_raw, Ring &r)
{
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    r.full = reinterpret_cast<uint64_t *>(smem + G::kBarOff);
    r.empty = r.full + S;
    r.accf = r.empty + S;
    r.acce = r.accf + 2;
    r.drain = r.acce + 2;
    r.holder = reinterpret_cast<uint32_t *>(smem + G::kMiscOff);
    r.abort_flag = reinterpret_cast<volatile int *>(smem + G::kMiscOff + 4);
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&r.full[s], 1);
            mbar_init(&r.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&r.accf[b], 1);
            mbar_init(&r.acce[b], 4);  // one arrival per epilogue warp
        }
        mbar_init(r.drain, 1);
        *r.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(r.holder, G::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return smem;
}

template <class G>
__device__ __forceinline__ void ring_teardown(uint32_t tmem)
{
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, G::kTmemCols);
    }
}

template <int S>
__device__ __forceinline__ void producer_drain(const Ring &r, int issued, const WaitCfg &wc)
{
    for (int it = issued > S ? issued - S : 0; it < issued; ++it)
        mbar_wait_drain(&r.full[it % S], (it / S) & 1, wc);
}

// MMA issue for one tile: nkb K-slices of 64; weight tile m of the stage accumulates into
// columns [d + m*BN, d + m*BN + n). Returns false if a wait gave up.
template <class G, int S, int BN, int MT>
__device__ __forceinline__ bool mma_tile(const Ring &r, uint8_t *smem, uint32_t d, int n, int nkb, int &it,
                                         const WaitCfg &wc)
{
    const uint32_t idesc = idesc_bf16_f32(128, n);
    for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % S;
        if (!mbar_wait(&r.full[s], (it / S) & 1, wc, r.abort_flag))
            return false;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * G::kStageBytes);
        const uint64_t bd = sdesc_kmajor_sw128(a_addr + G::kABytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint64_t ad = sdesc_kmajor_sw128(a_addr + m * kATileBytes);
                umma_bf16(d + m * BN, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
            }
        }
        umma_commit(&r.empty[s]);
    }
    return true;
}

// ------------------------------------------------------------------------------------
// gate_up: h[slot, f] = act(Wg_e[f]·x[tok], Wu_e[f]·x[tok]) for one chunk of an expert.
// A weight tile = 64 (gate, up) row pairs of one expert, interleaved by the 4-D tensor
// map (H, half, row, expert) so TMEM lane 2i holds gate row i and lane 2i+1 its up row;
// the epilogue pairs them with one shuffle. A tile covers MT * 64 features. Routed
// chunks read x_perm; the shared expert's chunks read x directly (identity permutation).
template <int BN, int S, int MT>
__global__ void __launch_bounds__(kThreads, 1)
    gate_up_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_wsh,
                   const __grid_constant__ CUtensorMap tm_xp, const __grid_constant__ CUtensorMap tm_x,
                   const GateUpArgs a, const WaitCfg wc)
{
    using G = Geo<BN, S, MT>;
    extern __shared__ uint8_t smem_raw[];
    Ring r;
    uint8_t *smem = ring_setup<G, S>(smem_raw, r);
    const uint32_t tmem = *r.holder;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int nrc, ntot;
    table_counts(a.hdr, a.max_chunks, a.err, nrc, ntot);
    const int tiles_r = nrc * (a.I / (64 * MT));
    const int tiles = tiles_r + (ntot - nrc) * (a.Is / (64 * MT));
    const int nkb = a.H / kBK;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_map(&tm_w);
            tma_prefetch_map(&tm_wsh);
            tma_prefetch_map(&tm_xp);
            tma_prefetch_map(&tm_x);
            int it = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < tiles && !stop; tile += gridDim.x) {
                int g, row0, ntok, fb;
                decode_gate_up<MT>(a, nrc, tiles_r, tile, g, row0, ntok, fb);
                const bool sh = g == a.E;
                const CUtensorMap *mw = sh ? &tm_wsh : &tm_w;
                const CUtensorMap *mb = sh ? &tm_x : &tm_xp;
                const int ge = sh ? 0 : g;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % S;
                    if (!mbar_wait(&r.empty[s], ((it / S) & 1) ^ 1, wc, r.abort_flag)) {
                        stop = true;
                        break;
                    }
                    // one box with the MT weight tiles, one box of BN token rows (rows past
                    // the chunk are loaded and ignored)
                    mbar_arrive_expect_tx(&r.full[s], G::kStageBytes);
                    uint8_t *A = smem + s * G::kStageBytes;
                    tma_load_4d(A, mw, &r.full[s], kb * kBK, 0, fb * MT * 64, ge);
                    tma_load_2d(A + G::kABytes, mb, &r.full[s], kb * kBK, row0);
                }
            }
            producer_drain<S>(r, it, wc);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int it = 0, tc = 0;
            for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
                int g, row0, ntok, fb;
                decode_gate_up<MT>(a, nrc, tiles_r, tile, g, row0, ntok, fb);
                const int buf = tc & 1;
                if (!mbar_wait(&r.acce[buf], ((tc >> 1) & 1) ^ 1, wc, r.abort_flag))
                    break;
                tc_fence_after();
                if (!mma_tile<G, S, BN, MT>(r, smem, tmem + buf * G::kBufCols, (ntok + 15) & ~15, nkb, it, wc))
                    break;
                umma_commit(&r.accf[buf]);
            }
            umma_commit(r.drain);
            mbar_wait_drain(r.drain, 0, wc);
        }
    } else {
        const int q = warp & 3;
        int tc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
            int g, row0, ntok, fb;
            decode_gate_up<MT>(a, nrc, tiles_r, tile, g, row0, ntok, fb);
            const int buf = tc & 1;
            if (!warp_wait(&r.accf[buf], (tc >> 1) & 1, wc, r.abort_flag))
                break;
            tc_fence_after();
            const bool sh = g == a.E;
            gate_up_epilogue<MT>(tmem + buf * G::kBufCols, BN, static_cast<int64_t>(fb) * MT * 64, ntok, row0,
                                 sh ? a.h_sh : a.h, sh ? a.Is : a.I, sh ? a.lim_s : a.lim_r, q, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&r.acce[buf]);
        }
    }
    ring_teardown<G>(tmem);
}

// ------------------------------------------------------------------------------------
// down: o[f, slot] = Wd_e[f]·h[slot]; routed slots add w_slot * o into y[token] (fp32
// atomics) or store it in o_perm[slot] (deterministic mode); shared rows add o (weight 1).
// A tile covers MT * 128 output features.
template <int BN, int S, int MT>
__global__ void __launch_bounds__(kThreads, 1)
    down_kernel(const __grid_constant__ CUtensorMap tm_wd, const __grid_constant__ CUtensorMap tm_wdsh,
                const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_hsh,
                const DownArgs a, const WaitCfg wc)
{
    using G = Geo<BN, S, MT>;
    extern __shared__ uint8_t smem_raw[];
    Ring r;
    uint8_t *smem = ring_setup<G, S>(smem_raw, r);
    const uint32_t tmem = *r.holder;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int nrc, ntot;
    table_counts(a.hdr, a.max_chunks, a.err, nrc, ntot);
    const int tiles = ntot * (a.H / (128 * MT));

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_map(&tm_wd);
            tma_prefetch_map(&tm_wdsh);
            tma_prefetch_map(&tm_h);
            tma_prefetch_map(&tm_hsh);
            int it = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < tiles && !stop; tile += gridDim.x) {
                int g, row0, ntok, fb;
                decode_down<MT>(a, tile, g, row0, ntok, fb);
                const bool sh = g == a.E;
                const int nkb = (sh ? a.Is : a.I) / kBK;
                const CUtensorMap *mw = sh ? &tm_wdsh : &tm_wd;
                const CUtensorMap *mb = sh ? &tm_hsh : &tm_h;
                const int wrow = (sh ? 0 : g * a.H) + fb * MT * 128;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % S;
                    if (!mbar_wait(&r.empty[s], ((it / S) & 1) ^ 1, wc, r.abort_flag)) {
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&r.full[s], G::kStageBytes);
                    uint8_t *A = smem + s * G::kStageBytes;
                    tma_load_2d(A, mw, &r.full[s], kb * kBK, wrow);
                    tma_load_2d(A + G::kABytes, mb, &r.full[s], kb * kBK, row0);
                }
            }
            producer_drain<S>(r, it, wc);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int it = 0, tc = 0;
            for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
                int g, row0, ntok, fb;
                decode_down<MT>(a, tile, g, row0, ntok, fb);
                const int nkb = (g == a.E ? a.Is : a.I) / kBK;
                const int buf = tc & 1;
                if (!mbar_wait(&r.acce[buf], ((tc >> 1) & 1) ^ 1, wc, r.abort_flag))
                    break;
                tc_fence_after();
                if (!mma_tile<G, S, BN, MT>(r, smem, tmem + buf * G::kBufCols, (ntok + 15) & ~15, nkb, it, wc))
                    break;
                umma_commit(&r.accf[buf]);
            }
            umma_commit(r.drain);
            mbar_wait_drain(r.drain, 0, wc);
        }
    } else {
        const int q = warp & 3;
        int tc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
            int g, row0, ntok, fb;
            decode_down<MT>(a, tile, g, row0, ntok, fb);
            const int buf = tc & 1;
            if (!warp_wait(&r.accf[buf], (tc >> 1) & 1, wc, r.abort_flag))
                break;
            tc_fence_after();
            down_epilogue<MT>(tmem + buf * G::kBufCols, BN, static_cast<int64_t>(fb) * MT * 128, ntok, row0,
                              g == a.E, a, q, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&r.acce[buf]);
        }
    }
    ring_teardown<G>(tmem);
}

template <int BN, int S, int MT>
cudaError_t gate_up_impl(const CUtensorMap &tm_w, const CUtensorMap &tm_wsh, const CUtensorMap &tm_xp,
                         const CUtensorMap &tm_x, const GateUpArgs &a, const WaitCfg &wc, int grid,
                         cudaStream_t stream)
{
    constexpr int smem = static_cast<int>(Geo<BN, S, MT>::kSmemBytes);
    cudaError_t err =
        cudaFuncSetAttribute(gate_up_kernel<BN, S, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    gate_up_kernel<BN, S, MT><<<grid, kThreads, smem, stream>>>(tm_w, tm_wsh, tm_xp, tm_x, a, wc);
    return cudaGetLastError();
}

template <int BN, int S, int MT>
cudaError_t down_impl(const CUtensorMap &tm_wd, const CUtensorMap &tm_wdsh, const CUtensorMap &tm_h,
                      const CUtensorMap &tm_hsh, const DownArgs &a, const WaitCfg &wc, int grid, cudaStream_t stream)
{
    constexpr int smem = static_cast<int>(Geo<BN, S, MT>::kSmemBytes);
    cudaError_t err = cudaFuncSetAttribute(down_kernel<BN, S, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    down_kernel<BN, S, MT><<<grid, kThreads, smem, stream>>>(tm_wd, tm_wdsh, tm_h, tm_hsh, a, wc);
    return cudaGetLastError();
}

}  // namespace

// Configurations (chosen by gemm_config): CTA pairs (expert_gemm_pair.cu); decode chunks
// of <= 32 tokens with one weight tile per stage and a 10-deep ring of 20 KB stages;
// chunks of <= 128 tokens with two weight tiles per stage (48 KB stages, 4 deep); shapes
// whose I, Is or H do not split into two tiles use one weight tile and <= 256 tokens.
cudaError_t launch_gate_up(const CUtensorMap &tm_w, const CUtensorMap &tm_wsh, const TokMaps &tok,
                           const GateUpArgs &a, const WaitCfg &wc, int grid, const GemmConfig &c,
                           cudaStream_t stream)
{
    if (c.pair)
        return launch_gate_up_pair(tm_w, tm_wsh, tok, a, wc, grid, stream);
    const CUtensorMap &tm_xp = tok.routed, &tm_x = tok.shared;
    if (c.cap == 32)
        return gate_up_impl<32, 10, 1>(tm_w, tm_wsh, tm_xp, tm_x, a, wc, grid, stream);
    if (c.mt == 2)
        return gate_up_impl<128, 4, 2>(tm_w, tm_wsh, tm_xp, tm_x, a, wc, grid, stream);
    return gate_up_impl<256, 4, 1>(tm_w, tm_wsh, tm_xp, tm_x, a, wc, grid, stream);
}

cudaError_t launch_down(const CUtensorMap &tm_wd, const CUtensorMap &tm_wdsh, const TokMaps &tok,
                        const DownArgs &a, const WaitCfg &wc, int grid, const GemmConfig &c, cudaStream_t stream)
{
    if (c.pair)
        return launch_down_pair(tm_wd, tm_wdsh, tok, a, wc, grid, stream);
    const CUtensorMap &tm_h = tok.routed, &tm_hsh = tok.shared;
    if (c.cap_d == 32)
        return down_impl<32, 10, 1>(tm_wd, tm_wdsh, tm_h, tm_hsh, a, wc, grid, stream);
    if (c.mt_d == 2)
        return down_impl<128, 4, 2>(tm_wd, tm_wdsh, tm_h, tm_hsh, a, wc, grid, stream);
    return down_impl<256, 4, 1>(tm_wd, tm_wdsh, tm_h, tm_hsh, a, wc, grid, stream);
}

}  // namespace moe
