// expert_gemm_pair.cu — grouped expert GEMMs on CTA pairs (tcgen05 cta_group::2).
//
// Same layer steps and layouts as expert_gemm.cu ("MAX 中 Step-3.5-Flash 架构解析",
// section "MoE共享专家、sigmoid 路由与激活裁剪": routed_moe(x) + shared_expert(x) with the
// clipped, concatenated gate/up activation), for prefill-sized calls. Two CTAs of a
// cluster (an SM pair) work on one tile: each holds MT weight tiles of 128 rows and HALF
// of the token rows of the chunk; the leader CTA issues M = 256 MMAs that read the weight
// rows of both CTAs and the token rows of both, and each CTA's TMEM receives its own 128
// weight rows x all N tokens. Per SM, the token bytes per stage halve, so more weight bytes
// are in flight (the HBM-bound case) and each MMA reads half as many token bytes from this
// SM's shared memory (the compute-bound case). gate_up stages hold two 64-wide K slices:
// the single MMA-issuing thread then pays its per-stage barrier test and commit once per
// 8 pair MMAs instead of 4.
//
// Pair protocol (leader = cluster rank 0):
//   - both producers load into their own shared memory; the transaction bytes of both
//     complete on the LEADER's full barrier, which only the leader arms (expect_tx);
//   - the leader's MMA commit arrives on the empty / accumulator-full / drain barriers of
//     both CTAs (multicast commit), so each producer and epilogue waits locally;
//   - both CTAs' epilogue warps arrive on the leader's accumulator-empty barrier (8 arrivals);
//   - TMEM is allocated and freed by warp 1 of both CTAs together (cta_group::2).
// Every mbarrier wait is bounded; the cluster barriers at the start and end are reached
// by every thread of both CTAs on every path.
#include "epilogue.cuh"

namespace moe {
namespace {

constexpr int kBK = 64;
constexpr uint32_t kATileBytes = 128 * 128;  // 128 weight rows x 64 bf16
// Token rows reach shared memory in boxes of 64 rows (8 KB per K slice); a stage loads only
// the boxes that hold rows of its chunk, so a short chunk in a wide tile costs no extra bytes.

// BN = token rows per pair tile (N of the pair MMA); each CTA holds BN/2 of them.
// NB = accumulator buffers in TMEM (2: the epilogue of one tile overlaps the next tile's
// mainloop; 1: larger tiles, the MMA waits for the epilogue between tiles).
// OUT = bytes of output staging after the ring (the down epilogue's bulk-reduction buffers).
// NSL = 64-wide K slices per stage, each laid out as [MT weight tiles][token rows]: more MMAs
// per barrier wait of the single MMA-issuing thread, fewer stages. Each slice has its own
// empty barrier: the MMA thread commits after each slice's MMAs, so the producer refills
// the first slice of a stage while the MMAs of the second are still running.
template <int BN, int S, int MT, int NB, int OUT = 0, int NSL = 1>
struct PairGeo {
    static constexpr uint32_t kABytes = MT * kATileBytes;
    static constexpr uint32_t kBBytes = (BN / 2) * 128;
    static constexpr uint32_t kSliceBytes = kABytes + kBBytes;
    static constexpr uint32_t kStageBytes = NSL * kSliceBytes;
    static constexpr uint32_t kOutOff = S * kStageBytes;
    static constexpr uint32_t kBarOff = kOutOff + OUT;
    // barriers: S full, S * NSL empty, 2 accumulator-full, 2 accumulator-empty, drain;
    // misc: TMEM holder, abort flag, then 8 epilogue flags per epilogue group (up to four)
    static constexpr int kNsl = NSL;
    static constexpr uint32_t kMiscOff = kBarOff + 8 * (S + S * NSL + 5);
    static constexpr uint32_t kSmemBytes = kMiscOff + 144 + 1024;
    static constexpr uint32_t kBufCols = MT * BN;
    static constexpr uint32_t kTmemCols = NB * kBufCols <= 32 ? 32 : (NB * kBufCols <= 64 ? 64 : (NB * kBufCols <= 128 ? 128 : (NB * kBufCols <= 256 ? 256 : 512)));
    static_assert(NB * kBufCols <= 512, "accumulators exceed TMEM");
    static_assert(kSliceBytes % 1024 == 0, "slices must stay 1024-byte aligned");
    static_assert(kSmemBytes <= kMaxDynSmem, "ring exceeds shared memory");

    static_assert(BN % 32 == 0 && BN <= 256, "pair token tile");
    static_assert(BN / 2 <= kPairTokBoxStep * kPairTokBoxes, "token rows per CTA fit the largest box");
};

struct PairRing {
    uint64_t *full, *empty, *accf, *acce, *drain;
    uint32_t *holder;
    volatile int *abort_flag;
    uint32_t rank;
    uint32_t full_leader;  // shared::cluster address of the leader's full[0]
    uint32_t acce_leader;  // shared::cluster address of the leader's acce[0]
};

// epi_warps: epilogue warps per CTA (each arrives once per tile on the leader's
// accumulator-empty barrier, from both CTAs).
template <class G, int S>
__device__ __forceinline__ uint8_t *pair_setup(uint8_t *smem_raw, PairRing &r, int epi_warps = 4)
{
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    r.full = reinterpret_cast<uint64_t *>(smem + G::kBarOff);
    r.empty = r.full + S;
    r.accf = r.empty + S * G::kNsl;
    r.acce = r.accf + 2;
    r.drain = r.acce + 2;
    r.holder = reinterpret_cast<uint32_t *>(smem + G::kMiscOff);
    r.abort_flag = reinterpret_cast<volatile int *>(smem + G::kMiscOff + 4);
    r.rank = cluster_ctarank();
    r.full_leader = dsmem_addr(smem_u32(r.full), 0);
    r.acce_leader = dsmem_addr(smem_u32(r.acce), 0);
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s)
            mbar_init(&r.full[s], 1);
        for (int s = 0; s < S * G::kNsl; ++s)
            mbar_init(&r.empty[s], 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&r.accf[b], 1);
            mbar_init(&r.acce[b], 2 * epi_warps);  // every epilogue warp of both CTAs
        }
        mbar_init(r.drain, 1);
        *r.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(r.holder, G::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs are initialised before any remote arrival
    tc_fence_after();
    return smem;
}

template <class G>
__device__ __forceinline__ void pair_teardown(uint32_t tmem)
{
    tc_fence_before();
    cluster_sync_all();  // both CTAs are done with TMEM, shared memory and each other's barriers
    if ((threadIdx.x >> 5) == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, G::kTmemCols);
    }
}

// On the way out the loads this CTA issued must have landed. The leader waits on its full
// barriers (both CTAs' bytes count there) for the last S stages it armed. The peer cannot
// wait on the leader's barriers; after a normal run its loads are the same stages the
// leader drains, but after an aborted run it may have issued stages the leader never
// armed, so it then waits 200 us (TMA latency is microseconds) before the final cluster
// barrier, behind which neither CTA exits.
template <int S>
__device__ __forceinline__ void pair_producer_drain(const PairRing &r, int issued, bool aborted, const WaitCfg &wc)
{
    if (r.rank != 0) {
        if (aborted) {
            const unsigned long long t0 = global_ns();
            while (global_ns() - t0 < 200000ull) {
            }
        }
        return;
    }
    for (int it = issued > S ? issued - S : 0; it < issued; ++it)
        mbar_wait_drain(&r.full[it % S], (it / S) & 1, wc);
}

// Leader's MMA issue for one pair tile: nkb stages of NSL 64-wide K slices; weight tile m
// accumulates into columns [d + m*BN, d + m*BN + n) of both CTAs' TMEM.
template <class G, int S, int BN, int MT, int NSL>
__device__ __forceinline__ bool pair_mma_tile(const PairRing &r, uint8_t *smem, uint32_t d, int n, int nkb,
                                              int &it, const WaitCfg &wc)
{
    const uint32_t idesc = idesc_bf16_f32(256, n);
    for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % S;
        if (!mbar_wait(&r.full[s], (it / S) & 1, wc, r.abort_flag))
            return false;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < NSL; ++c) {
            const uint32_t a_addr = smem_u32(smem + s * G::kStageBytes + c * G::kSliceBytes);
            const uint64_t bd = sdesc_kmajor_sw128(a_addr + G::kABytes);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint64_t ad = sdesc_kmajor_sw128(a_addr + m * kATileBytes);
                    umma_bf16_pair(d + m * BN, ad + 2 * kk, bd + 2 * kk, idesc, (kb | c | kk) != 0);
                }
            }
            umma_commit_pair_mc(&r.empty[s * NSL + c], 0x3);  // this slice's buffers are free
        }
    }
    return true;
}

// The leader runs the MMA loop; the peer's MMA warp only waits for the final drain.
template <class G, int S, int BN, int MT, int NB, int NSL, class NextTile>
__device__ __forceinline__ void pair_mma_role(const PairRing &r, uint8_t *smem, uint32_t tmem, int first,
                                              int tiles, int stride, NextTile tile_info, const WaitCfg &wc)
{
    if (r.rank == 0) {
        int it = 0, tc = 0;
        for (int tile = first; tile < tiles; tile += stride, ++tc) {
            int ntok, nkb;
            tile_info(tile, ntok, nkb);
            const int buf = tc % NB;
            if (!mbar_wait(&r.acce[buf], ((tc / NB) & 1) ^ 1, wc, r.abort_flag))
                break;
            tc_fence_after();
            if (!pair_mma_tile<G, S, BN, MT, NSL>(r, smem, tmem + buf * G::kBufCols, (ntok + 15) & ~15, nkb, it,
                                                  wc))
                break;
            umma_commit_pair_mc(&r.accf[buf], 0x3);
        }
        umma_commit_pair_mc(r.drain, 0x3);
    }
    mbar_wait_drain(r.drain, 0, wc);
}

// ------------------------------------------------------------------------------------
// gate_up on pairs: a pair tile covers 2 * MT * 64 features (CTA r holds weight tiles
// (fb * 2 + r) * MT + m of 64 (gate, up) row pairs each).
template <int MT>
__device__ __forceinline__ void decode_gate_up_pair(const GateUpArgs &a, int nrc, int tiles_r, int tile, int &g,
                                                    int &row0, int &ntok, int &fb)
{
    int ci;
    if (tile < tiles_r) {
        const int nfb = a.I / (128 * MT);
        ci = tile / nfb;
        fb = tile - ci * nfb;
    } else {
        const int nfb = a.Is / (128 * MT);
        const int tt = tile - tiles_r;
        ci = nrc + tt / nfb;
        fb = tt - (tt / nfb) * nfb;
    }
    const int4 c = chunk_at(a, ci);
    g = c.x;
    row0 = c.y;
    ntok = c.z;
}

// EW epilogue warps (4 or 8): with 8, two warps share each TMEM lane quarter and take
// alternate 32-column blocks of the tile.
template <int BN, int S, int MT, int NB, int NSL, int EW>
__global__ void __launch_bounds__(64 + 32 * EW, 1)
    gate_up_pair_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_wsh,
                        const __grid_constant__ PairTokMaps tok, const GateUpArgs a, const WaitCfg wc)
{
    static_assert(EW % 4 == 0 && EW >= 4 && EW <= 16, "one to four groups of four epilogue warps");
    using G = PairGeo<BN, S, MT, NB, 0, NSL>;
    extern __shared__ uint8_t smem_raw[];
    PairRing r;
    uint8_t *smem = pair_setup<G, S>(smem_raw, r, EW);
    const uint32_t tmem = *r.holder;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int nrc, ntot;
    table_counts(a.hdr, a.max_chunks, a.err, nrc, ntot);
    const int tiles_r = nrc * (a.I / (128 * MT));
    const int tiles = tiles_r + (ntot - nrc) * (a.Is / (128 * MT));
    const int nkb = a.H / (kBK * NSL);  // stages per tile
    const int first = blockIdx.x >> 1;
    const int stride = gridDim.x >> 1;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_map(&tm_w);
            tma_prefetch_map(&tm_wsh);
            for (int i = 0; i < kPairTokBoxes; ++i) {
                tma_prefetch_map(&tok.routed_b[i]);
                tma_prefetch_map(&tok.shared_b[i]);
            }
            int it = 0;
            bool stop = false;
            for (int tile = first; tile < tiles && !stop; tile += stride) {
                int g, row0, ntok, fb;
                decode_gate_up_pair<MT>(a, nrc, tiles_r, tile, g, row0, ntok, fb);
                const bool sh = g == a.E;
                const int half = ((ntok + 15) & ~15) >> 1;  // token rows used from each CTA
                // one token box per K slice: the smallest box height covering the half
                const int bi = (half + kPairTokBoxStep - 1) / kPairTokBoxStep - 1;
                const uint32_t tok_bytes = (bi + 1) * kPairTokBoxStep * 128;
                const CUtensorMap *mw = sh ? &tm_wsh : &tm_w;
                const CUtensorMap *mb = sh ? &tok.shared_b[bi] : &tok.routed_b[bi];
                const int ge = sh ? 0 : g;
                const int wt0 = (fb * 2 + static_cast<int>(r.rank)) * MT;
                const int brow = row0 + static_cast<int>(r.rank) * half;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % S;
                    const uint32_t par = ((it / S) & 1) ^ 1;
                    if (!mbar_wait(&r.empty[s * NSL], par, wc, r.abort_flag)) {
                        stop = true;
                        break;
                    }
                    if (r.rank == 0)
                        mbar_arrive_expect_tx(&r.full[s], 2 * NSL * (G::kABytes + tok_bytes));
                    const uint32_t bar = r.full_leader + 8 * s;
                    // per K slice, once its buffers are free: one box with this CTA's MT
                    // weight tiles, then one box of token rows covering its half of the chunk
                    // (rows past the half are loaded and ignored)
                    for (int c = 0; c < NSL; ++c) {
                        if (c > 0 && !mbar_wait(&r.empty[s * NSL + c], par, wc, r.abort_flag)) {
                            stop = true;
                            break;
                        }
                        uint8_t *A = smem + s * G::kStageBytes + c * G::kSliceBytes;
                        const int k0 = (kb * NSL + c) * kBK;
                        tma_load_4d_pair(A, mw, bar, k0, 0, wt0 * 64, ge);
                        tma_load_2d_pair(A + G::kABytes, mb, bar, k0, brow);
                    }
                    if (stop) {
                        ++it;  // a partly issued stage: the drain also waits for its copies
                        break;
                    }
                }
            }
            pair_producer_drain<S>(r, it, stop || *r.abort_flag, wc);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            auto info = [&](int tile, int &ntok, int &nk) {
                int g, row0, fb;
                decode_gate_up_pair<MT>(a, nrc, tiles_r, tile, g, row0, ntok, fb);
                nk = nkb;
            };
            pair_mma_role<G, S, BN, MT, NB, NSL>(r, smem, tmem, first, tiles, stride, info, wc);
        }
    } else {
        const int q = warp & 3;
        const int grp = (warp - 2) / 4;
        int tc = 0;
        for (int tile = first; tile < tiles; tile += stride, ++tc) {
            int g, row0, ntok, fb;
            decode_gate_up_pair<MT>(a, nrc, tiles_r, tile, g, row0, ntok, fb);
            const int buf = tc % NB;
            if (!warp_wait(&r.accf[buf], (tc / NB) & 1, wc, r.abort_flag))
                break;
            tc_fence_after();
            const bool sh = g == a.E;
            const int wt0 = (fb * 2 + static_cast<int>(r.rank)) * MT;
            gate_up_epilogue<MT>(tmem + buf * G::kBufCols, BN, static_cast<int64_t>(wt0) * 64, ntok, row0,
                                 sh ? a.h_sh : a.h, sh ? a.Is : a.I, sh ? a.lim_s : a.lim_r, q, lane, grp * 32,
                                 (EW / 4) * 32);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(r.acce_leader + 8 * buf);
        }
    }
    pair_teardown<G>(tmem);
}

// ------------------------------------------------------------------------------------
// down on pairs: a pair tile covers 2 * MT * 128 output features.
//
// Epilogue through shared memory and TMA bulk reductions: per block of 16 token columns,
// the four warps of an epilogue group write the weighted outputs of this CTA's MT * 128
// features as 16 rows of MT * 512 bytes (one row per token) into a staging buffer; then one
// lane per token issues a bulk reduce-add of its row into y[token] (or, in deterministic
// mode, a bulk store into o_perm[slot]). Each output row thus takes one MT * 512-byte
// reduction at L2 instead of MT * 4 reductions of 128 bytes. NOB staging buffers per group
// rotate so a block's reductions overlap the next block's TMEM loads; a buffer is
// rewritten only after its bulk reads are done. With EW = 8 epilogue warps, two groups of
// four (each covering all 128 TMEM lanes) take alternate 16-token blocks of a tile, with
// their own staging buffers and named barrier (id 1 + group).
constexpr int kOutTok = 16;

template <int MT, int NOB>
__device__ __forceinline__ void down_epilogue_bulk(uint32_t tmem_tile, int bn, int64_t feat0, int ntok, int64_t row0,
                                                   bool sh, const DownArgs &a, int q, int lane, uint8_t *stage,
                                                   int &ob, int grp, int ngrp)
{
    constexpr uint32_t kRowBytes = MT * 128 * 4;
    constexpr uint32_t kBufBytes = kOutTok * kRowBytes;
    const int bar_id = 1 + grp;
    for (int cb = grp * kOutTok; cb < ntok; cb += ngrp * kOutTok, ++ob) {
        uint8_t *buf = stage + (ob % NOB) * kBufBytes;
        // lane l (and l + 16) fetch the destination row and weight of column cb + l % 16
        // (-1: no column)
        const int mycol = cb + (lane & (kOutTok - 1));
        int64_t dst_row = -1;
        float wgt = 0.0f;
        if (mycol < ntok) {
            const int64_t rr = row0 + mycol;
            if (!down_dst_row(a, sh, rr, dst_row))
                dst_row = -1;
            wgt = sh ? 1.0f : a.w_perm[rr];
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float v[kOutTok];
            tmem_load16(tmem_tile + m * bn + (static_cast<uint32_t>(q * 32) << 16) + cb, v);
            float *col = reinterpret_cast<float *>(buf) + m * 128 + q * 32 + lane;
#pragma unroll
            for (int i = 0; i < kOutTok; ++i)
                col[i * (kRowBytes / 4)] = __shfl_sync(0xFFFFFFFFu, wgt, i) * v[i];
        }
        fence_proxy_async_smem();
        named_bar_sync(bar_id, 128);
        if (q == 0 && lane < kOutTok) {
            if (dst_row >= 0) {
                float *dst = a.out + dst_row * a.H + feat0;
                // each output row receives k + 1 reductions spread over the whole launch:
                // keep its lines in L2 against the weight stream (evict-last policy)
                if (a.deterministic)
                    bulk_store(dst, buf + lane * kRowBytes, kRowBytes);
                else
                    bulk_reduce_add_f32_hint(dst, buf + lane * kRowBytes, kRowBytes, l2_policy_evict_last());
                bulk_commit();
            }
            bulk_wait_read<NOB - 1>();  // the buffer written next is no longer being read
        }
        named_bar_sync(bar_id, 128);
    }
}
template <int MT>
__device__ __forceinline__ void decode_down_pair(const DownArgs &a, int tile, int &g, int &row0, int &ntok, int &fb)
{
    const int nfb = a.H / (256 * MT);
    const int ci = tile / nfb;
    fb = tile - ci * nfb;
    const int4 c = chunk_at(a, ci);
    g = c.x;
    row0 = c.y;
    ntok = c.z;
}

// BN token rows per tile (BN / 2 per CTA), S stages of NSL 64-wide K slices, MT weight
// tiles of 128 rows per CTA and slice, NB TMEM accumulators, NOB staging buffers per
// epilogue group, EW epilogue warps (4 or 8).
template <int BN, int S, int MT, int NB, int NOB, int NSL, int EW>
__global__ void __launch_bounds__(64 + 32 * EW, 1)
    down_pair_kernel(const __grid_constant__ CUtensorMap tm_wd, const __grid_constant__ CUtensorMap tm_wdsh,
                     const __grid_constant__ PairTokMaps tok, const DownArgs a, const WaitCfg wc)
{
    static_assert(EW % 4 == 0 && EW >= 4 && EW <= 16, "one to four groups of four epilogue warps");
    constexpr int kGroups = EW / 4;
    using G = PairGeo<BN, S, MT, NB, kGroups * NOB * kOutTok * MT * 512, NSL>;
    extern __shared__ uint8_t smem_raw[];
    PairRing r;
    uint8_t *smem = pair_setup<G, S>(smem_raw, r, EW);
    const uint32_t tmem = *r.holder;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int nrc, ntot;
    table_counts(a.hdr, a.max_chunks, a.err, nrc, ntot);
    const int tiles = ntot * (a.H / (256 * MT));
    const int first = blockIdx.x >> 1;
    const int stride = gridDim.x >> 1;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_map(&tm_wd);
            tma_prefetch_map(&tm_wdsh);
            for (int i = 0; i < kPairTokBoxes; ++i) {
                tma_prefetch_map(&tok.routed_b[i]);
                tma_prefetch_map(&tok.shared_b[i]);
            }
            int it = 0;
            bool stop = false;
            for (int tile = first; tile < tiles && !stop; tile += stride) {
                int g, row0, ntok, fb;
                decode_down_pair<MT>(a, tile, g, row0, ntok, fb);
                const bool sh = g == a.E;
                const int nkb = (sh ? a.Is : a.I) / (kBK * NSL);
                const int half = ((ntok + 15) & ~15) >> 1;
                const int bi = (half + kPairTokBoxStep - 1) / kPairTokBoxStep - 1;
                const uint32_t tok_bytes = (bi + 1) * kPairTokBoxStep * 128;
                const CUtensorMap *mw = sh ? &tm_wdsh : &tm_wd;
                const CUtensorMap *mb = sh ? &tok.shared_b[bi] : &tok.routed_b[bi];
                const int wrow = (sh ? 0 : g * a.H) + (fb * 2 + static_cast<int>(r.rank)) * MT * 128;
                const int brow = row0 + static_cast<int>(r.rank) * half;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % S;
                    const uint32_t par = ((it / S) & 1) ^ 1;
                    if (!mbar_wait(&r.empty[s * NSL], par, wc, r.abort_flag)) {
                        stop = true;
                        break;
                    }
                    if (r.rank == 0)
                        mbar_arrive_expect_tx(&r.full[s], 2 * NSL * (G::kABytes + tok_bytes));
                    const uint32_t bar = r.full_leader + 8 * s;
                    for (int c = 0; c < NSL; ++c) {
                        if (c > 0 && !mbar_wait(&r.empty[s * NSL + c], par, wc, r.abort_flag)) {
                            stop = true;
                            break;
                        }
                        uint8_t *A = smem + s * G::kStageBytes + c * G::kSliceBytes;
                        const int k0 = (kb * NSL + c) * kBK;
                        tma_load_2d_pair(A, mw, bar, k0, wrow);
                        tma_load_2d_pair(A + G::kABytes, mb, bar, k0, brow);
                    }
                    if (stop) {
                        ++it;  // a partly issued stage: the drain also waits for its copies
                        break;
                    }
                }
            }
            pair_producer_drain<S>(r, it, stop || *r.abort_flag, wc);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            auto info = [&](int tile, int &ntok, int &nk) {
                int g, row0, fb;
                decode_down_pair<MT>(a, tile, g, row0, ntok, fb);
                nk = (g == a.E ? a.Is : a.I) / (kBK * NSL);
            };
            pair_mma_role<G, S, BN, MT, NB, NSL>(r, smem, tmem, first, tiles, stride, info, wc);
        }
    } else {
        const int q = warp & 3;
        const int grp = (warp - 2) / 4;
        const int bar_id = 1 + grp;
        int tc = 0, ob = 0;
        volatile int *epi_ok = reinterpret_cast<volatile int *>(smem + G::kMiscOff + 16) + grp * 8;
        uint8_t *stage = smem + G::kOutOff + grp * (NOB * kOutTok * MT * 512);
        for (int tile = first; tile < tiles; tile += stride, ++tc) {
            int g, row0, ntok, fb;
            decode_down_pair<MT>(a, tile, g, row0, ntok, fb);
            const int buf = tc % NB;
            // The four warps of a group agree on the wait's outcome before the
            // barrier-synchronised epilogue, so a wait that expires in one warp cannot
            // strand the others at a named barrier (flags double-buffered by tile parity).
            const bool ok = warp_wait(&r.accf[buf], (tc / NB) & 1, wc, r.abort_flag);
            if (lane == 0)
                epi_ok[(tc & 1) * 4 + q] = ok ? 1 : 0;
            named_bar_sync(bar_id, 128);
            const volatile int *f = epi_ok + (tc & 1) * 4;
            if (!(f[0] && f[1] && f[2] && f[3]))
                break;
            tc_fence_after();
            const int wt0 = (fb * 2 + static_cast<int>(r.rank)) * MT;
            down_epilogue_bulk<MT, NOB>(tmem + buf * G::kBufCols, BN, static_cast<int64_t>(wt0) * 128, ntok, row0,
                                        g == a.E, a, q, lane, stage, ob, grp, kGroups);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(r.acce_leader + 8 * buf);
        }
        if (q == 0 && lane < kOutTok)
            bulk_wait<0>();  // this lane's reductions have landed before the CTA exits
    }
    pair_teardown<G>(tmem);
}

PairTokMaps pair_maps(const TokMaps &t)
{
    PairTokMaps p;
    for (int i = 0; i < kPairTokBoxes; ++i) {
        p.routed_b[i] = t.routed_b[i];
        p.shared_b[i] = t.shared_b[i];
    }
    return p;
}

// Launches `grid` CTAs (rounded down to pairs) as clusters of 2, but no more pairs than can be
// resident at once (cudaOccupancyMaxActiveClusters): the kernels are persistent, so a pair that
// could only start after another one exits would run its whole tile share as a tail.
template <class Kernel, class... Args>
cudaError_t launch_pairs(Kernel kernel, int smem, int grid, int threads, cudaStream_t stream, Args... args)
{
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid & ~1, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int resident = 0;
    err = cudaOccupancyMaxActiveClusters(&resident, kernel, &cfg);
    if (err != cudaSuccess)
        return err;
    if (resident < 1)
        return cudaErrorInvalidConfiguration;
    if (2 * resident < static_cast<int>(cfg.gridDim.x))
        cfg.gridDim.x = 2 * resident;
    err = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (err != cudaSuccess)
        return err;
    return cudaGetLastError();
}

// gate_up: pair tiles of up to 256 token rows (128 per CTA) x 128 features, one weight
// tile per CTA and K slice, two 64-wide K slices per stage (8 pair MMAs per barrier test
// and commit of the MMA thread), three 64 KB stages. Most experts of a prefill batch then
// need one pass over their weights. down: the same 256-row chunks x 256 output features, one
// weight tile per CTA and K slice, two K slices per stage (three 64 KB stages), sixteen
// epilogue warps in four groups, each with one 8 KB output staging buffer for the bulk
// reductions. The down epilogue is bound by the reductions it keeps in flight: a 256-column
// tile's K loop (I = 1536) is short against its 128 KB of fp32 output per CTA. Measured on
// the Step-5 shapes against 128-row chunks with two weight tiles per CTA and four epilogue
// warps: 256-row chunks with 4 warps 20-35% slower, with 8 warps (two buffers each) 5%
// faster, with 16 warps 10-14% faster; 12 or 16 warps adding straight from registers
// (coalesced fp32 reductions, no staging) 5-11%; 24 warps on a 5 x 32 KB ring slower. Both
// keep two TMEM accumulators.
constexpr int kGateUpStages = 3, kGateUpSlices = 2, kGateUpBufs = 2, kGateUpEpiWarps = 4;
using GateUpPair = PairGeo<kPairCapGateUp, kGateUpStages, kPairMtGateUp, kGateUpBufs, 0, kGateUpSlices>;
constexpr int kDownStages = 3, kDownSlices = 2, kDownOutBufs = 1, kDownEpiWarps = 16;
using DownPair = PairGeo<kPairCapDown, kDownStages, kPairMtDown, 2,
                         (kDownEpiWarps / 4) * kDownOutBufs * kOutTok * kPairMtDown * 512, kDownSlices>;

}  // namespace

cudaError_t launch_gate_up_pair(const CUtensorMap &tm_w, const CUtensorMap &tm_wsh, const TokMaps &tok,
                                const GateUpArgs &a, const WaitCfg &wc, int grid, cudaStream_t stream)
{
    return launch_pairs(gate_up_pair_kernel<kPairCapGateUp, kGateUpStages, kPairMtGateUp, kGateUpBufs, kGateUpSlices,
                                            kGateUpEpiWarps>,
                        static_cast<int>(GateUpPair::kSmemBytes), grid, 64 + 32 * kGateUpEpiWarps, stream, tm_w,
                        tm_wsh, pair_maps(tok), a, wc);
}

cudaError_t launch_down_pair(const CUtensorMap &tm_wd, const CUtensorMap &tm_wdsh, const TokMaps &tok,
                             const DownArgs &a, const WaitCfg &wc, int grid, cudaStream_t stream)
{
    return launch_pairs(
        down_pair_kernel<kPairCapDown, kDownStages, kPairMtDown, 2, kDownOutBufs, kDownSlices, kDownEpiWarps>,
        static_cast<int>(DownPair::kSmemBytes), grid, 64 + 32 * kDownEpiWarps, stream, tm_wd, tm_wdsh, pair_maps(tok),
        a, wc);
}

}  // namespace moe
