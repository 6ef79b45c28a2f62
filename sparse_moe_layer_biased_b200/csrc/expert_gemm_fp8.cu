// expert_gemm_fp8.cu — grouped expert GEMMs with FP8 E4M3 routed-expert weights.
//
// Weight format: miles Step-5-Preview page, section 1 ("FP8 checkpoint"): the routed
// experts are stored in FP8 E4M3 with one scale per 128x128 block and are dequantized
// on load; the shared expert stays BF16. The layer steps are those of expert_gemm.cu
// ("MAX 中 Step-3.5-Flash 架构解析", section "MoE共享专家、sigmoid 路由与激活裁剪").
//
// Dequantization happens on the way from HBM to the tensor cores. A deep staging ring
// receives, per K slice, the E4M3 weight tile (64 bytes per row, half the bytes of
// BF16) and the token rows; four converter warps turn the weight tile into
// bf16(e4m3 * block_scale) in the 128-byte-swizzled K-major layout the MMA reads, in a
// shallow ring of converted tiles; the MMA (the BF16 tcgen05 MMA of the BF16 path) reads
// the converted tile and the token rows straight from the staging slot, then frees both
// slots. Loads therefore run a whole staging ring ahead of the MMA, and the converted
// ring's turnaround holds no memory latency. Shared-expert tiles are BF16: their weight
// tile lands directly in the converted ring.
//
// Roles per CTA (persistent, one CTA per SM, static round-robin over tiles):
//   warp 0      staging producer: E4M3 weight tile (routed experts) + token rows
//   warp 1      MMA issuer and TMEM owner (2 accumulator buffers)
//   warps 2..5  epilogue (TMEM -> activation / weighting -> global)
//   warps 6..9  converters: staged E4M3 tile -> converted bf16 tile, one block scale per
//               128-row weight group and 128-wide K block
//   warp 10     shared-expert producer: BF16 weight tiles of the shared expert -> converted ring
// Every wait is bounded; on expiry the CTA drains its own copies and MMAs, frees TMEM
// and returns with the device error word set.
#include <cuda_fp8.h>

#include "epilogue.cuh"

namespace moe {
namespace {

constexpr int kThreads8 = 352;
constexpr int kBK = 64;
constexpr uint32_t kATileBytes = 128 * 128;  // 128 weight rows x 64 bf16 (converted)
constexpr uint32_t kQTileBytes = 128 * 64;   // 128 weight rows x 64 E4M3 codes (staged)

// BN token rows per chunk, SW staging slots (MT E4M3 weight tiles + BN token rows),
// SA converted slots (MT bf16 weight tiles).
template <int BN, int SA, int SW, int MT>
struct Geo8 {
    static constexpr uint32_t kABytes = MT * kATileBytes;  // converted slot
    static constexpr uint32_t kQBytes = MT * kQTileBytes;  // staged E4M3 part of a staging slot
    static constexpr uint32_t kBBytes = BN * 128;          // token part of a staging slot
    static constexpr uint32_t kQSlotBytes = kQBytes + kBBytes;
    static constexpr uint32_t kQOff = SA * kABytes;
    static constexpr uint32_t kBarOff = kQOff + SW * kQSlotBytes;
    static constexpr uint32_t kNumBars = 2 * SW + 3 * SA + 5;
    static constexpr uint32_t kMiscOff = kBarOff + 8 * kNumBars;
    static constexpr uint32_t kSmemBytes = kMiscOff + 16 + 1024;
    static constexpr uint32_t kBufCols = MT * BN;
    static constexpr uint32_t kTmemCols = 2 * kBufCols < 32 ? 32 : 2 * kBufCols;
    static_assert(kABytes % 1024 == 0 && kQSlotBytes % 1024 == 0 && kQBytes % 1024 == 0,
                  "slots stay 1024-byte aligned");
    static_assert(kSmemBytes <= kMaxDynSmem, "rings exceed shared memory");
    static_assert((kTmemCols & (kTmemCols - 1)) == 0 && kTmemCols <= 512, "TMEM allocation");
};

struct Ring8 {
    uint64_t *qfull, *qempty;        // staging ring: bytes landed / MMA done with the slot
    uint64_t *afull, *conv, *aempty;  // converted ring: shared-expert weights landed (or a
                                      // plain arrival) / converted / MMA done with the slot
    uint64_t *accf, *acce, *drain;
    uint32_t *holder;
    volatile int *abort_flag;
};

template <class G, int SA, int SW>
__device__ __forceinline__ uint8_t *ring8_setup(uint8_t *smem_raw, Ring8 &r)
{
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    r.qfull = reinterpret_cast<uint64_t *>(smem + G::kBarOff);
    r.qempty = r.qfull + SW;
    r.afull = r.qempty + SW;
    r.conv = r.afull + SA;
    r.aempty = r.conv + SA;
    r.accf = r.aempty + SA;
    r.acce = r.accf + 2;
    r.drain = r.acce + 2;
    r.holder = reinterpret_cast<uint32_t *>(smem + G::kMiscOff);
    r.abort_flag = reinterpret_cast<volatile int *>(smem + G::kMiscOff + 4);
    if (threadIdx.x == 0) {
        for (int s = 0; s < SW; ++s) {
            mbar_init(&r.qfull[s], 1);
            mbar_init(&r.qempty[s], 1);
        }
        for (int s = 0; s < SA; ++s) {
            mbar_init(&r.afull[s], 1);
            mbar_init(&r.conv[s], 4);  // one arrival per converter warp
            mbar_init(&r.aempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&r.accf[b], 1);
            mbar_init(&r.acce[b], 4);  // one arrival per epilogue warp
        }
        mbar_init(r.drain, 1);
        *r.abort_flag = 0;
        fence_barrier_init();
    }
    if ((threadIdx.x >> 5) == 1) {
        tmem_alloc(r.holder, G::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return smem;
}

template <class G>
__device__ __forceinline__ void ring8_teardown(uint32_t tmem)
{
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, G::kTmemCols);
    }
}

// Waits for the last `depth` phases of `bars` that this role armed (its own copies).
__device__ __forceinline__ void drain_ring(uint64_t *bars, int depth, int issued, const WaitCfg &wc)
{
    for (int it = issued > depth ? issued - depth : 0; it < issued; ++it)
        mbar_wait_drain(&bars[it % depth], (it / depth) & 1, wc);
}

// bf16 pair (lo, hi) of e4m3 codes b0 (lower K) and b1, each times `scale`.
__device__ __forceinline__ uint32_t dequant2(uint32_t codes16, float scale)
{
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(codes16), __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * scale, f.y * scale);
    return *reinterpret_cast<const uint32_t *>(&b);
}

// Converts one staged weight tile (128 rows x 64 E4M3 codes, row j at j * 64 bytes) into
// the 128-byte-swizzled K-major bf16 tile the MMA reads (row j at (j / 8) * 1024 +
// (j % 8) * 128, 16-byte chunk c stored at chunk c ^ (j % 8)). Row j takes scale
// s_odd when j is odd, else s_even (gate_up tiles interleave gate and up rows, which
// sit in different 128-row scale blocks). The 128 converter threads each take 4 units
// of 16 codes; a warp reads 512 contiguous staged bytes per step.
__device__ __forceinline__ void convert_tile(const uint8_t *q, uint8_t *a, float s_even, float s_odd, int ct)
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int u = ct + 128 * i;
        const int j = u >> 2, c = u & 3;
        const uint4 v = *reinterpret_cast<const uint4 *>(q + j * 64 + c * 16);
        const float s = (j & 1) ? s_odd : s_even;
        uint4 lo, hi;
        lo.x = dequant2(v.x & 0xFFFFu, s);
        lo.y = dequant2(v.x >> 16, s);
        lo.z = dequant2(v.y & 0xFFFFu, s);
        lo.w = dequant2(v.y >> 16, s);
        hi.x = dequant2(v.z & 0xFFFFu, s);
        hi.y = dequant2(v.z >> 16, s);
        hi.z = dequant2(v.w & 0xFFFFu, s);
        hi.w = dequant2(v.w >> 16, s);
        uint8_t *row = a + (j >> 3) * 1024 + (j & 7) * 128;
        *reinterpret_cast<uint4 *>(row + (((2 * c) ^ (j & 7)) << 4)) = lo;
        *reinterpret_cast<uint4 *>(row + (((2 * c + 1) ^ (j & 7)) << 4)) = hi;
    }
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// One tile of either GEMM: group g (E = shared expert), chunk rows [row0, row0 + ntok),
// feature block fb, nkb K slices.
struct Tile8 {
    int g, row0, ntok, fb, nkb;
    bool sh;
};

template <int MT>
__device__ __forceinline__ Tile8 tile_of(const GateUpArgs &a, int tile)
{
    const int nrc = a.hdr[0];
    const int tiles_r = nrc * (a.I / (64 * MT));
    Tile8 t;
    decode_gate_up<MT>(a, nrc, tiles_r, tile, t.g, t.row0, t.ntok, t.fb);
    t.sh = t.g == a.E;
    t.nkb = a.H / kBK;
    return t;
}

template <int MT>
__device__ __forceinline__ Tile8 tile_of(const DownArgs &a, int tile)
{
    Tile8 t;
    decode_down<MT>(a, tile, t.g, t.row0, t.ntok, t.fb);
    t.sh = t.g == a.E;
    t.nkb = (t.sh ? a.Is : a.I) / kBK;
    return t;
}

template <int MT>
__device__ __forceinline__ int tile_count(const GateUpArgs &a)
{
    const int nrc = a.hdr[0];
    return nrc * (a.I / (64 * MT)) + (a.hdr[1] - nrc) * (a.Is / (64 * MT));
}

template <int MT>
__device__ __forceinline__ int tile_count(const DownArgs &a)
{
    return a.hdr[1] * (a.H / (128 * MT));
}

// Weight tile(s) of K slice kb: gate_up maps are (H, half, row, expert) with boxes of
// MT*64 (gate, up) row pairs; down maps are (I, rows) with boxes of MT*128 rows.
template <int MT>
__device__ __forceinline__ void load_weights(const GateUpArgs &a, const CUtensorMap *m, void *dst, uint64_t *bar,
                                             const Tile8 &t, int kb)
{
    tma_load_4d(dst, m, bar, kb * kBK, 0, t.fb * MT * 64, t.sh ? 0 : t.g);
}

template <int MT>
__device__ __forceinline__ void load_weights(const DownArgs &a, const CUtensorMap *m, void *dst, uint64_t *bar,
                                             const Tile8 &t, int kb)
{
    tma_load_2d(dst, m, bar, kb * kBK, (t.sh ? 0 : t.g * a.H) + t.fb * MT * 128);
}

// Block scales of weight tile m at K slice kb (even rows, odd rows). gate_up tile m holds
// gate rows f0 .. f0+63 (scale row block f0/128) interleaved with up rows I+f0 .. (block
// (I+f0)/128), f0 = (fb*MT + m)*64; scales [E, 2I/128, H/128].
template <int MT>
__device__ __forceinline__ float2 tile_scales(const GateUpArgs &a, const Tile8 &t, int m, int kb)
{
    const int nbr = a.I / 64, nbc = a.H / 128;
    const float *srow = a.w_scale + static_cast<int64_t>(t.g) * nbr * nbc + kb / 2;
    const int f0 = (t.fb * MT + m) * 64;
    return make_float2(__ldg(srow + static_cast<int64_t>(f0 / 128) * nbc),
                       __ldg(srow + static_cast<int64_t>((a.I + f0) / 128) * nbc));
}

// down tile m holds output rows (fb*MT + m)*128 .. +127, one scale row block; scales
// [E, H/128, I/128].
template <int MT>
__device__ __forceinline__ float2 tile_scales(const DownArgs &a, const Tile8 &t, int m, int kb)
{
    const int nbr = a.H / 128, nbc = a.I / 128;
    const float v = __ldg(a.w_scale + (static_cast<int64_t>(t.g) * nbr + t.fb * MT + m) * nbc + kb / 2);
    return make_float2(v, v);
}

template <int MT>
__device__ __forceinline__ void epilogue8(const GateUpArgs &a, uint32_t tmem_tile, int bn, const Tile8 &t, int q,
                                          int lane)
{
    gate_up_epilogue<MT>(tmem_tile, bn, static_cast<int64_t>(t.fb) * MT * 64, t.ntok, t.row0, t.sh ? a.h_sh : a.h,
                         t.sh ? a.Is : a.I, t.sh ? a.lim_s : a.lim_r, q, lane);
}

template <int MT>
__device__ __forceinline__ void epilogue8(const DownArgs &a, uint32_t tmem_tile, int bn, const Tile8 &t, int q,
                                          int lane)
{
    down_epilogue<MT>(tmem_tile, bn, static_cast<int64_t>(t.fb) * MT * 128, t.ntok, t.row0, t.sh, a, q, lane);
}

// ------------------------------------------------------------------------------------
// Both GEMMs with E4M3 routed weights. Maps: m_w (E4M3 codes), m_wsh (BF16 shared
// weights), m_tok (routed token rows: x_perm or h), m_tok_sh (shared token rows: x or
// h_sh). Stage `it` uses staging slot it % SW and converted slot it % SA.
template <class Args, int BN, int SA, int SW, int MT>
__global__ void __launch_bounds__(kThreads8, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap m_w, const __grid_constant__ CUtensorMap m_wsh,
                    const __grid_constant__ CUtensorMap m_tok, const __grid_constant__ CUtensorMap m_tok_sh,
                    const Args a, const WaitCfg wc)
{
    using G = Geo8<BN, SA, SW, MT>;
    extern __shared__ uint8_t smem_raw[];
    Ring8 r;
    uint8_t *smem = ring8_setup<G, SA, SW>(smem_raw, r);
    const uint32_t tmem = *r.holder;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tiles = tile_count<MT>(a);
    uint8_t *const conv_ring = smem;
    uint8_t *const stage_ring = smem + G::kQOff;

    if (warp == 0) {
        // staging producer: E4M3 weights (routed) and token rows, one slot per K slice
        if (lane == 0) {
            tma_prefetch_map(&m_w);
            tma_prefetch_map(&m_tok);
            tma_prefetch_map(&m_tok_sh);
            int it = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < tiles && !stop; tile += gridDim.x) {
                const Tile8 t = tile_of<MT>(a, tile);
                for (int kb = 0; kb < t.nkb; ++kb, ++it) {
                    const int s = it % SW;
                    if (!mbar_wait(&r.qempty[s], ((it / SW) & 1) ^ 1, wc, r.abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *slot = stage_ring + s * G::kQSlotBytes;
                    mbar_arrive_expect_tx(&r.qfull[s], G::kBBytes + (t.sh ? 0u : G::kQBytes));
                    if (!t.sh)
                        load_weights<MT>(a, &m_w, slot, &r.qfull[s], t, kb);
                    tma_load_2d(slot + G::kQBytes, t.sh ? &m_tok_sh : &m_tok, &r.qfull[s], kb * kBK, t.row0);
                }
            }
            drain_ring(r.qfull, SW, it, wc);
        }
    } else if (warp == 10) {
        // shared-expert BF16 weights straight into the converted ring; routed slots get a
        // plain arrival so every converted slot completes one afull phase per stage
        if (lane == 0) {
            tma_prefetch_map(&m_wsh);
            int it = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < tiles && !stop; tile += gridDim.x) {
                const Tile8 t = tile_of<MT>(a, tile);
                for (int kb = 0; kb < t.nkb; ++kb, ++it) {
                    const int s = it % SA;
                    if (!mbar_wait(&r.aempty[s], ((it / SA) & 1) ^ 1, wc, r.abort_flag)) {
                        stop = true;
                        break;
                    }
                    if (t.sh) {
                        mbar_arrive_expect_tx(&r.afull[s], G::kABytes);
                        load_weights<MT>(a, &m_wsh, conv_ring + s * G::kABytes, &r.afull[s], t, kb);
                    } else {
                        mbar_arrive(&r.afull[s]);
                    }
                }
            }
            drain_ring(r.afull, SA, it, wc);
        }
    } else if (warp >= 6) {
        // converters: stage `it` is ready for the MMA once its staged bytes landed and
        // (routed) its weight tile is converted or (shared) its BF16 tile landed
        const int ct = threadIdx.x - 192;
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            const Tile8 t = tile_of<MT>(a, tile);
            for (int kb = 0; kb < t.nkb; ++kb, ++it) {
                const int sa = it % SA, sq = it % SW;
                ok = warp_wait(&r.aempty[sa], ((it / SA) & 1) ^ 1, wc, r.abort_flag) &&
                     warp_wait(&r.qfull[sq], (it / SW) & 1, wc, r.abort_flag) &&
                     warp_wait(&r.afull[sa], (it / SA) & 1, wc, r.abort_flag);
                if (!ok)
                    break;
                if (!t.sh) {
                    const uint8_t *q = stage_ring + sq * G::kQSlotBytes;
                    uint8_t *dst = conv_ring + sa * G::kABytes;
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const float2 sc = tile_scales<MT>(a, t, m, kb);
                        convert_tile(q + m * kQTileBytes, dst + m * kATileBytes, sc.x, sc.y, ct);
                    }
                    fence_proxy_async_smem();  // generic-proxy stores -> the MMA's async-proxy reads
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&r.conv[sa]);
            }
        }
    } else if (warp == 1) {
        // MMA: converted weights (A) x staged token rows (B); one commit frees both slots
        if (lane == 0) {
            int it = 0, tc = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tc) {
                const Tile8 t = tile_of<MT>(a, tile);
                const int buf = tc & 1;
                if (!mbar_wait(&r.acce[buf], ((tc >> 1) & 1) ^ 1, wc, r.abort_flag))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + buf * G::kBufCols;
                const uint32_t idesc = idesc_bf16_f32(128, (t.ntok + 15) & ~15);
                for (int kb = 0; kb < t.nkb; ++kb, ++it) {
                    const int sa = it % SA, sq = it % SW;
                    if (!mbar_wait(&r.conv[sa], (it / SA) & 1, wc, r.abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(conv_ring + sa * G::kABytes);
                    const uint64_t bd = sdesc_kmajor_sw128(smem_u32(stage_ring + sq * G::kQSlotBytes) + G::kQBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            const uint64_t ad = sdesc_kmajor_sw128(a_addr + m * kATileBytes);
                            umma_bf16(d + m * BN, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                        }
                    }
                    umma_commit(&r.aempty[sa]);
                    umma_commit(&r.qempty[sq]);
                }
                if (ok)
                    umma_commit(&r.accf[buf]);
            }
            umma_commit(r.drain);
            mbar_wait_drain(r.drain, 0, wc);
        }
    } else {
        // warps 2..5: epilogue
        const int q = warp & 3;
        int tc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
            const Tile8 t = tile_of<MT>(a, tile);
            const int buf = tc & 1;
            if (!warp_wait(&r.accf[buf], (tc >> 1) & 1, wc, r.abort_flag))
                break;
            tc_fence_after();
            epilogue8<MT>(a, tmem + buf * G::kBufCols, BN, t, q, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&r.acce[buf]);
        }
    }
    ring8_teardown<G>(tmem);
}

template <class Args, int BN, int SA, int SW, int MT>
cudaError_t launch8(int grid, cudaStream_t stream, const CUtensorMap &m0, const CUtensorMap &m1,
                    const CUtensorMap &m2, const CUtensorMap &m3, const Args &a, const WaitCfg &wc)
{
    constexpr int smem = static_cast<int>(Geo8<BN, SA, SW, MT>::kSmemBytes);
    auto kernel = gemm_fp8_kernel<Args, BN, SA, SW, MT>;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    kernel<<<grid, kThreads8, smem, stream>>>(m0, m1, m2, m3, a, wc);
    return cudaGetLastError();
}

}  // namespace

// Decode-sized calls: 32-row chunks; 12 KB staging slots (8 KB E4M3 + 4 KB tokens), 12
// deep (96 KB of weight bytes in flight per SM), 4 converted slots of 16 KB. Prefill:
// 128-row chunks; 24 KB staging slots, 7 deep; 3 converted slots.
cudaError_t launch_gate_up_fp8(const CUtensorMap &tm_w, const CUtensorMap &tm_wsh, const CUtensorMap &tm_xp,
                               const CUtensorMap &tm_x, const GateUpArgs &a, const WaitCfg &wc, int grid,
                               const GemmConfig &c, cudaStream_t stream)
{
    if (c.cap == 32)
        return launch8<GateUpArgs, 32, 4, 12, 1>(grid, stream, tm_w, tm_wsh, tm_xp, tm_x, a, wc);
    return launch8<GateUpArgs, 128, 3, 7, 1>(grid, stream, tm_w, tm_wsh, tm_xp, tm_x, a, wc);
}

cudaError_t launch_down_fp8(const CUtensorMap &tm_wd, const CUtensorMap &tm_wdsh, const CUtensorMap &tm_h,
                            const CUtensorMap &tm_hsh, const DownArgs &a, const WaitCfg &wc, int grid,
                            const GemmConfig &c, cudaStream_t stream)
{
    if (c.cap_d == 32)
        return launch8<DownArgs, 32, 4, 12, 1>(grid, stream, tm_wd, tm_wdsh, tm_h, tm_hsh, a, wc);
    return launch8<DownArgs, 128, 3, 7, 1>(grid, stream, tm_wd, tm_wdsh, tm_h, tm_hsh, a, wc);
}

}  // namespace moe
