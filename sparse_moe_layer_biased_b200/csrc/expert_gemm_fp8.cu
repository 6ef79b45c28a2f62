// expert_gemm_fp8.cu — grouped expert GEMMs with FP8 E4M3 routed-expert weights.
//
// Weight format: miles Step-5-Preview page, section 1 ("FP8 checkpoint"): the routed
// experts are stored in FP8 E4M3 with one scale per 128x128 block and are dequantized
// on load; the shared expert stays BF16. The layer steps are those of expert_gemm.cu
// ("MAX 中 Step-3.5-Flash 架构解析", section "MoE共享专家、sigmoid 路由与激活裁剪").
//
// Dequantization happens on the way from HBM to the tensor cores without a second trip
// through shared memory. A staging ring receives, per pipeline stage, the weight tile of
// 128 rows and the token rows: a routed stage spans one 128-wide scale block (E4M3 codes,
// 128 bytes per row: half the bytes of BF16), a shared-expert stage 64 K elements of its
// BF16 weights (also 128 bytes per row). Converter warps each take one weight row (one
// TMEM lane), turn it into bf16(e4m3 * block_scale) and store it into a TMEM operand
// slot; the BF16 tcgen05 MMA reads A from TMEM and the token rows (B) from the staging
// slot. Shared memory then carries each weight byte once in and once out, fewer bytes
// per weight element than the BF16 kernels move. Two groups of four converter warps take
// alternate stages, so one group's conversion overlaps the other's waits; a tile's block
// scales are read once per tile into registers.
//
// Roles per CTA (persistent, one CTA per SM, static round-robin over tiles):
//   warp 0       staging producer: weight tile (E4M3 routed / BF16 shared) + token rows
//   warp 1       MMA issuer and TMEM owner (2 accumulator buffers, SA operand slots)
//   warps 2..5   epilogue (TMEM -> activation / weighting -> global)
//   warps 6..13  converters, group 0 (warps 6..9) on even stages, group 1 on odd ones;
//                warp w handles weight rows / TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31
// Every wait is bounded; on expiry the CTA drains its own copies and MMAs, frees TMEM
// and returns with the device error word set.
#include <cuda_bf16.h>

#include "epilogue.cuh"

namespace moe {
namespace {

constexpr int kThreads8 = 448;
constexpr int kBK = 64;
constexpr uint32_t kWBytes = 128 * 128;  // weight part of a staging slot: 128 rows x 128 bytes
constexpr uint32_t kACols = 64;          // TMEM columns of one operand slot: 128 bf16 per row

// BN token rows per chunk, SW staging slots, SA TMEM operand slots, KS 128-wide scale
// blocks per stage (a routed stage spans 128 KS of K, a shared-expert stage 64 KS).
template <int BN, int SW, int SA, int KS>
struct Geo8 {
    static constexpr uint32_t kBSlice = BN * 128;  // token rows of one 64-wide K slice
    static constexpr uint32_t kWStage = KS * kWBytes;
    static constexpr uint32_t kSlotBytes = kWStage + 2 * KS * kBSlice;
    static constexpr uint32_t kSlotCols = KS * kACols;  // TMEM columns of one operand slot
    static constexpr uint32_t kBarOff = SW * kSlotBytes;
    static constexpr uint32_t kNumBars = 2 * SW + 2 * SA + 5;
    static constexpr uint32_t kMiscOff = kBarOff + 8 * kNumBars;
    static constexpr uint32_t kSmemBytes = kMiscOff + 16 + 1024;
    static constexpr uint32_t kBufCols = BN;             // one accumulator buffer
    static constexpr uint32_t kAOff = 2 * kBufCols;      // first operand slot column
    static constexpr uint32_t kUsedCols = kAOff + SA * kSlotCols;
    static constexpr uint32_t kTmemCols = kUsedCols <= 128 ? 128 : (kUsedCols <= 256 ? 256 : 512);
    static_assert(kSlotBytes % 1024 == 0, "slots stay 1024-byte aligned");
    static_assert(kSmemBytes <= kMaxDynSmem, "ring exceeds shared memory");
    static_assert(kUsedCols <= 512, "accumulators and operand slots exceed TMEM");
};

struct Ring8 {
    uint64_t *qfull, *qempty;  // staging ring: bytes landed / MMA done with the slot
    uint64_t *conv, *aempty;   // TMEM operand slots: converted / MMA done with the slot
    uint64_t *accf, *acce, *drain;
    uint32_t *holder;
    volatile int *abort_flag;
};

template <class G, int SW, int SA>
__device__ __forceinline__ uint8_t *ring8_setup(uint8_t *smem_raw, Ring8 &r)
{
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    r.qfull = reinterpret_cast<uint64_t *>(smem + G::kBarOff);
    r.qempty = r.qfull + SW;
    r.conv = r.qempty + SW;
    r.aempty = r.conv + SA;
    r.accf = r.aempty + SA;
    r.acce = r.accf + 2;
    r.drain = r.acce + 2;
    r.holder = reinterpret_cast<uint32_t *>(smem + G::kMiscOff);
    r.abort_flag = reinterpret_cast<volatile int *>(smem + G::kMiscOff + 4);
    // equal ring depths: stage it uses staging slot and operand slot it % SW, both freed by
    // the same MMA completion, so one barrier (one commit per stage) releases both
    if (SA == SW)
        r.aempty = r.qempty;
    if (threadIdx.x == 0) {
        for (int s = 0; s < SW; ++s) {
            mbar_init(&r.qfull[s], 1);
            mbar_init(&r.qempty[s], 1);
        }
        for (int s = 0; s < SA; ++s) {
            mbar_init(&r.conv[s], 4);  // one arrival per warp of the converting group
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

// Dequantization on the integer and FMA pipes. An E4M3 code s.eeee.mmm placed in a bf16
// word as s.0000eeee.mmm0000 (sign at bit 15, exponent field e, fraction m/8) is a bf16
// number whose value is exactly the code's value times 2^-120: normal codes map to bf16
// normals 2^(e-127)(1 + m/8) = 2^-120 * 2^(e-7)(1 + m/8), subnormal codes to bf16
// subnormals 2^-126 * m/8 = 2^-120 * 2^-6 * m/8. The block scale then multiplies as
// S = scale * 2^120 (exact in fp32 for |scale| < 2^8), split into bf16 parts
// S = S_hi + S_lo: the weight is fma(q, S_hi, q * S_lo), within one bf16 ulp of
// bf16(code value * scale) (equal to it except near rounding ties: the S_lo product
// carries a relative error of 2^-18). The two E4M3 NaN codes are not decoded as NaN
// (checkpoints hold none).
struct Scale2 {
    __nv_bfloat162 hi, lo;
};

__device__ __forceinline__ Scale2 split_scale(float scale)
{
    const float S = scale * 0x1p120f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(S);
    const __nv_bfloat16 lo = __float2bfloat16_rn(S - __bfloat162float(hi));
    return Scale2{__bfloat162bfloat162(hi), __bfloat162bfloat162(lo)};
}

// Codes (b0, b1) of the byte pair `sel` selects (0x4140: bytes 0, 1; 0x4342: bytes 2, 3)
// -> bf16x2 (low half = lower K) of code value * scale. Each code lands in bits 0..7 of its
// 16-bit half; multiplying by 16 moves it to bits 4..11, and adding 240 x (its sign bit)
// carries the sign from bit 11 to bit 15 (2^11 + 15 * 2^11 = 2^15), so the integer work is
// one byte permute, one mask and one multiply-add.
__device__ __forceinline__ uint32_t dequant2(uint32_t codes4, uint32_t sel, const Scale2 &sc)
{
    const uint32_t pu = __byte_perm(codes4, 0u, sel);
    const uint32_t sg = pu & 0x00800080u;
    const uint32_t bits = pu * 16u + sg * 240u;
    const __nv_bfloat162 q = *reinterpret_cast<const __nv_bfloat162 *>(&bits);
    const __nv_bfloat162 w = __hfma2(q, sc.hi, __hmul2(q, sc.lo));
    return *reinterpret_cast<const uint32_t *>(&w);
}

// Byte offset of 16-byte chunk c of row j in a 128-byte-swizzled tile of 128-byte rows
// (the TMA SWIZZLE_128B layout: chunk c of row j stored at chunk c ^ (j % 8)).
__device__ __forceinline__ uint32_t sw128_chunk(int j, int c)
{
    return static_cast<uint32_t>((j >> 3) * 1024 + (j & 7) * 128 + ((c ^ (j & 7)) << 4));
}

// Routed stage: converts row j (128 E4M3 codes) of the staged tile and stores the 64
// bf16 pairs into TMEM lane j, columns taddr .. taddr + 63 (taddr carries the lane).
__device__ __forceinline__ void convert_row_e4m3(const uint8_t *w, int j, uint32_t taddr, const Scale2 &s)
{
#pragma unroll
    for (int h = 0; h < 4; ++h) {  // 32 codes -> 16 columns per store
        uint32_t out[16];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const uint4 v = *reinterpret_cast<const uint4 *>(w + sw128_chunk(j, 2 * h + cc));
            out[8 * cc + 0] = dequant2(v.x, 0x4140u, s);
            out[8 * cc + 1] = dequant2(v.x, 0x4342u, s);
            out[8 * cc + 2] = dequant2(v.y, 0x4140u, s);
            out[8 * cc + 3] = dequant2(v.y, 0x4342u, s);
            out[8 * cc + 4] = dequant2(v.z, 0x4140u, s);
            out[8 * cc + 5] = dequant2(v.z, 0x4342u, s);
            out[8 * cc + 6] = dequant2(v.w, 0x4140u, s);
            out[8 * cc + 7] = dequant2(v.w, 0x4342u, s);
        }
        tmem_store16(taddr + 16 * h, out);
    }
}

// Shared-expert stage: copies row j (64 bf16) of the staged BF16 tile into TMEM lane j,
// columns taddr .. taddr + 31.
__device__ __forceinline__ void copy_row_bf16(const uint8_t *w, int j, uint32_t taddr)
{
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t out[16];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const uint4 v = *reinterpret_cast<const uint4 *>(w + sw128_chunk(j, 4 * h + cc));
            out[4 * cc + 0] = v.x;
            out[4 * cc + 1] = v.y;
            out[4 * cc + 2] = v.z;
            out[4 * cc + 3] = v.w;
        }
        tmem_store16(taddr + 16 * h, out);
    }
}

// One tile of either GEMM: group g (E = shared expert), chunk rows [row0, row0 + ntok),
// weight block fb (64 gate/up feature pairs, or 128 down rows), K extent K.
struct Tile8 {
    int g, row0, ntok, fb, K;
    bool sh;
    // K of one 128-byte weight box: a 128-wide scale block of E4M3 codes, or 64 K of the
    // BF16 shared expert; a stage holds KS boxes
    __device__ __forceinline__ int box_k() const { return sh ? 64 : 128; }
    __device__ __forceinline__ int stages(int ks) const { return (K + ks * box_k() - 1) / (ks * box_k()); }
};

__device__ __forceinline__ Tile8 tile_of(const GateUpArgs &a, int tile)
{
    int nrc, ntot;
    table_counts(a.hdr, a.max_chunks, a.err, nrc, ntot);
    Tile8 t;
    decode_gate_up<1>(a, nrc, nrc * (a.I / 64), tile, t.g, t.row0, t.ntok, t.fb);
    t.sh = t.g == a.E;
    t.K = a.H;
    return t;
}

__device__ __forceinline__ Tile8 tile_of(const DownArgs &a, int tile)
{
    Tile8 t;
    decode_down<1>(a, tile, t.g, t.row0, t.ntok, t.fb);
    t.sh = t.g == a.E;
    t.K = t.sh ? a.Is : a.I;
    return t;
}

__device__ __forceinline__ int tile_count(const GateUpArgs &a)
{
    int nrc, ntot;
    table_counts(a.hdr, a.max_chunks, a.err, nrc, ntot);
    return nrc * (a.I / 64) + (ntot - nrc) * (a.Is / 64);
}

__device__ __forceinline__ int tile_count(const DownArgs &a)
{
    int nrc, ntot;
    table_counts(a.hdr, a.max_chunks, a.err, nrc, ntot);
    return ntot * (a.H / 128);
}

// Weight box of one tile at K element k0 (128 rows x 128 bytes). gate_up maps are (K,
// half, row, expert) with boxes of 64 (gate, up) row pairs; down maps are (K, rows).
__device__ __forceinline__ void load_weights(const GateUpArgs &a, const CUtensorMap *m, void *dst, uint64_t *bar,
                                             const Tile8 &t, int k0)
{
    tma_load_4d(dst, m, bar, k0, 0, t.fb * 64, t.sh ? 0 : t.g);
}

__device__ __forceinline__ void load_weights(const DownArgs &a, const CUtensorMap *m, void *dst, uint64_t *bar,
                                             const Tile8 &t, int k0)
{
    tma_load_2d(dst, m, bar, k0, (t.sh ? 0 : t.g * a.H) + t.fb * 128);
}

// Block scales of a routed tile at 128-wide K block kblk: (even rows, odd rows). gate_up
// tile fb holds gate rows f0 .. f0+63 (scale row block f0/128) interleaved with up rows
// I+f0 .. (block (I+f0)/128), f0 = 64 fb; scales [E, 2I/128, H/128]. down tile fb holds
// rows 128 fb .. +127, one scale row block; scales [E, H/128, I/128].
__device__ __forceinline__ float2 tile_scales(const GateUpArgs &a, const Tile8 &t, int kblk)
{
    const int nbr = a.I / 64, nbc = a.H / 128;
    const float *srow = a.w_scale + static_cast<int64_t>(t.g) * nbr * nbc + kblk;
    const int f0 = t.fb * 64;
    return make_float2(__ldg(srow + static_cast<int64_t>(f0 / 128) * nbc),
                       __ldg(srow + static_cast<int64_t>((a.I + f0) / 128) * nbc));
}

__device__ __forceinline__ float2 tile_scales(const DownArgs &a, const Tile8 &t, int kblk)
{
    const int nbr = a.H / 128, nbc = a.I / 128;
    const float v = __ldg(a.w_scale + (static_cast<int64_t>(t.g) * nbr + t.fb) * nbc + kblk);
    return make_float2(v, v);
}

__device__ __forceinline__ void epilogue8(const GateUpArgs &a, uint32_t tmem_tile, int bn, const Tile8 &t, int q,
                                          int lane)
{
    gate_up_epilogue<1>(tmem_tile, bn, static_cast<int64_t>(t.fb) * 64, t.ntok, t.row0, t.sh ? a.h_sh : a.h,
                        t.sh ? a.Is : a.I, t.sh ? a.lim_s : a.lim_r, q, lane);
}

__device__ __forceinline__ void epilogue8(const DownArgs &a, uint32_t tmem_tile, int bn, const Tile8 &t, int q,
                                          int lane)
{
    down_epilogue<1>(tmem_tile, bn, static_cast<int64_t>(t.fb) * 128, t.ntok, t.row0, t.sh, a, q, lane);
}

// ------------------------------------------------------------------------------------
// Both GEMMs with E4M3 routed weights. Maps: m_w (E4M3 codes, 128-byte swizzled boxes of
// 128 K), m_wsh (BF16 shared weights, 64 K), m_tok (routed token rows: x_perm or h),
// m_tok_sh (shared token rows: x or h_sh). Stage `it` uses staging slot it % SW and TMEM
// operand slot it % SA; K elements past a tile's extent are zero-filled by TMA for both
// operands.
template <class Args, int BN, int SW, int SA, int KS>
__global__ void __launch_bounds__(kThreads8, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap m_w, const __grid_constant__ CUtensorMap m_wsh,
                    const __grid_constant__ CUtensorMap m_tok, const __grid_constant__ CUtensorMap m_tok_sh,
                    const Args a, const WaitCfg wc)
{
    using G = Geo8<BN, SW, SA, KS>;
    extern __shared__ uint8_t smem_raw[];
    Ring8 r;
    uint8_t *smem = ring8_setup<G, SW, SA>(smem_raw, r);
    const uint32_t tmem = *r.holder;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tiles = tile_count(a);

    if (warp == 0) {
        // staging producer: one weight box and one (shared) or two (routed) token slices
        if (lane == 0) {
            tma_prefetch_map(&m_w);
            tma_prefetch_map(&m_wsh);
            tma_prefetch_map(&m_tok);
            tma_prefetch_map(&m_tok_sh);
            int it = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < tiles && !stop; tile += gridDim.x) {
                const Tile8 t = tile_of(a, tile);
                const int nsl = (t.sh ? 1 : 2) * KS;  // 64-wide token slices per stage
                const int nst = t.stages(KS);
                for (int st = 0; st < nst; ++st, ++it) {
                    const int s = it % SW;
                    if (!mbar_wait(&r.qempty[s], ((it / SW) & 1) ^ 1, wc, r.abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *slot = smem + s * G::kSlotBytes;
                    const int k0 = st * KS * t.box_k();
                    mbar_arrive_expect_tx(&r.qfull[s], G::kWStage + nsl * G::kBSlice);
                    for (int c = 0; c < KS; ++c)
                        load_weights(a, t.sh ? &m_wsh : &m_w, slot + c * kWBytes, &r.qfull[s], t, k0 + c * t.box_k());
                    for (int kc = 0; kc < nsl; ++kc)
                        tma_load_2d(slot + G::kWStage + kc * G::kBSlice, t.sh ? &m_tok_sh : &m_tok, &r.qfull[s],
                                    k0 + kc * kBK, t.row0);
                }
            }
            drain_ring(r.qfull, SW, it, wc);
        }
    } else if (warp >= 6) {
        // converters: group gi takes the stages with it % 2 == gi; thread = weight row j
        const int gi = (warp - 6) >> 2;
        const int j = 32 * (warp & 3) + lane;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            const Tile8 t = tile_of(a, tile);
            const int nkblk = (t.K + 127) / 128;
            const int nst = t.stages(KS);
            // lane l caches the scales of K block base + l (reloaded every 32 blocks)
            int base = -32;
            float se = 0.0f, so = 0.0f;
            for (int st = 0; st < nst; ++st, ++it) {
                if ((it & 1) != gi)
                    continue;
                const int sa = it % SA, sq = it % SW;
                if (!t.sh && st * KS + KS - 1 - base >= 32) {
                    base = st * KS;
                    se = so = 0.0f;
                    if (base + lane < nkblk) {
                        const float2 sc = tile_scales(a, t, base + lane);
                        se = sc.x;
                        so = sc.y;
                    }
                }
                ok = warp_wait(&r.aempty[sa], ((it / SA) & 1) ^ 1, wc, r.abort_flag) &&
                     warp_wait(&r.qfull[sq], (it / SW) & 1, wc, r.abort_flag);
                if (!ok)
                    break;
                tc_fence_after();  // the MMA that read this operand slot has completed
#pragma unroll
                for (int c = 0; c < KS; ++c) {
                    const uint8_t *w = smem + sq * G::kSlotBytes + c * kWBytes;
                    const uint32_t taddr = lane_addr + G::kAOff + sa * G::kSlotCols;
                    if (t.sh) {
                        copy_row_bf16(w, j, taddr + c * (kACols / 2));
                    } else {
                        const float s_even = __shfl_sync(0xFFFFFFFFu, se, st * KS + c - base);
                        const float s_odd = __shfl_sync(0xFFFFFFFFu, so, st * KS + c - base);
                        convert_row_e4m3(w, j, taddr + c * kACols, split_scale((j & 1) ? s_odd : s_even));
                    }
                }
                tmem_store_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&r.conv[sa]);
            }
        }
    } else if (warp == 1) {
        // MMA: A (weights) from the TMEM operand slot, B (token rows) from the staging slot.
        // The converter group of a stage waited for the slot's bytes before it arrived on
        // conv, so conv's completion implies qfull's: the MMA thread waits on conv alone
        // (each barrier test costs the single issuing thread about 100 cycles per stage).
        if (lane == 0) {
            int it = 0, tc = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tc) {
                const Tile8 t = tile_of(a, tile);
                const int buf = tc & 1;
                if (!mbar_wait(&r.acce[buf], ((tc >> 1) & 1) ^ 1, wc, r.abort_flag))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + buf * G::kBufCols;
                const uint32_t idesc = idesc_bf16_f32(128, (t.ntok + 15) & ~15);
                const int nks = KS * t.box_k() / 16;  // K=16 MMAs per stage
                const int nst = t.stages(KS);
                for (int st = 0; st < nst; ++st, ++it) {
                    const int sa = it % SA, sq = it % SW;
                    if (!mbar_wait(&r.conv[sa], (it / SA) & 1, wc, r.abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_col = tmem + G::kAOff + sa * G::kSlotCols;
                    const uint32_t b_addr = smem_u32(smem + sq * G::kSlotBytes) + G::kWStage;
                    for (int ks = 0; ks < nks; ++ks) {
                        const uint64_t bd = sdesc_kmajor_sw128(b_addr + (ks >> 2) * G::kBSlice) + 2 * (ks & 3);
                        umma_bf16_ta(d, a_col + 8 * ks, bd, idesc, (st | ks) != 0);
                    }
                    if (SA != SW)
                        umma_commit(&r.aempty[sa]);
                    umma_commit(&r.qempty[sq]);
                }
                if (ok)
                    umma_commit(&r.accf[buf]);
            }
            umma_commit(r.drain);
            mbar_wait_drain(r.drain, 0, wc);
        }
    } else if (warp >= 2) {
        // warps 2..5: epilogue
        const int q = warp & 3;
        int tc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
            const Tile8 t = tile_of(a, tile);
            const int buf = tc & 1;
            if (!warp_wait(&r.accf[buf], (tc >> 1) & 1, wc, r.abort_flag))
                break;
            tc_fence_after();
            epilogue8(a, tmem + buf * G::kBufCols, BN, t, q, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&r.acce[buf]);
        }
    }
    ring8_teardown<G>(tmem);
}

template <class Args, int BN, int SW, int SA, int KS>
cudaError_t launch8(int grid, cudaStream_t stream, const CUtensorMap &m0, const CUtensorMap &m1,
                    const CUtensorMap &m2, const CUtensorMap &m3, const Args &a, const WaitCfg &wc)
{
    constexpr int smem = static_cast<int>(Geo8<BN, SW, SA, KS>::kSmemBytes);
    auto kernel = gemm_fp8_kernel<Args, BN, SW, SA, KS>;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    kernel<<<grid, kThreads8, smem, stream>>>(m0, m1, m2, m3, a, wc);
    return cudaGetLastError();
}

}  // namespace

// Decode-sized calls whose shapes the FP8 tensor-core kernels do not take (H not a multiple of
// 256, or I, Is not multiples of 128): 32-row chunks; stages of two scale blocks (256 K: 16 MMAs per barrier
// test and commit of the MMA thread), staging slots of 48 KB (32 KB weights + four 4 KB token
// slices), 4 deep; 3 TMEM operand slots of 128 columns.
// Prefill: 128-row chunks; stages of one scale block, 48 KB staging slots, 4 deep; 4 TMEM
// operand slots.
cudaError_t launch_gate_up_fp8(const CUtensorMap &tm_w, const CUtensorMap &tm_wsh, const CUtensorMap &tm_xp,
                               const CUtensorMap &tm_x, const GateUpArgs &a, const WaitCfg &wc, int grid,
                               const GemmConfig &c, cudaStream_t stream)
{
    if (c.cap == 32)
        return launch8<GateUpArgs, 32, 4, 3, 2>(grid, stream, tm_w, tm_wsh, tm_xp, tm_x, a, wc);
    return launch8<GateUpArgs, 128, 4, 4, 1>(grid, stream, tm_w, tm_wsh, tm_xp, tm_x, a, wc);
}

cudaError_t launch_down_fp8(const CUtensorMap &tm_wd, const CUtensorMap &tm_wdsh, const CUtensorMap &tm_h,
                            const CUtensorMap &tm_hsh, const DownArgs &a, const WaitCfg &wc, int grid,
                            const GemmConfig &c, cudaStream_t stream)
{
    if (c.cap_d == 32)
        return launch8<DownArgs, 32, 4, 3, 2>(grid, stream, tm_wd, tm_wdsh, tm_h, tm_hsh, a, wc);
    return launch8<DownArgs, 128, 4, 4, 1>(grid, stream, tm_wd, tm_wdsh, tm_h, tm_hsh, a, wc);
}

}  // namespace moe
