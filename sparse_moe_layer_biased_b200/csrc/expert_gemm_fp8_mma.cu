// expert_gemm_fp8_mma.cu — grouped expert GEMMs of decode-sized calls with FP8 E4M3
// routed-expert weights, multiplied on the FP8 tensor-core path (tcgen05 kind::f8f6f4).
//
// Weight format: miles Step-5-Preview page, section 1 ("FP8 checkpoint"): E4M3 codes with one
// fp32 scale per 128x128 block; the shared expert stays BF16. Layer steps: "MAX 中
// Step-3.5-Flash 架构解析", section "MoE共享专家、sigmoid 路由与激活裁剪".
//
// The weight codes go from HBM into shared memory by TMA and into the MMA as they are: no
// work per weight element. The block scale moves to the token operand instead, which at
// decode holds 16 or 32 rows per 128 weight rows. A tile is two 128-row weight blocks (for
// gate_up the gate rows f0 .. f0+127 and the matching up rows; for down 256 consecutive
// output rows), each with its own block scale row and TMEM accumulator. For 128-wide K block
// kb of weight block b the token-prep warps form, for token row j of the chunk,
//     v = x * s_b[kb] * 2^-e_b * 2^(6 - e_j)
// in fp32 (e_b = exponent of the largest scale of the block row, e_j = exponent of the
// row's largest |x|, so |v| < 2^8 <= the E4M3 maximum 448) and split it into two E4M3
// operands, hi = e4m3(v) and lo = e4m3(v - hi), stacked as rows [0, n) and [n, 2n) of one
// B operand (n = the chunk's rows rounded up to 16). One kind::f8f6f4 MMA per 32 K then
// produces W·hi and W·lo in neighbouring accumulator columns; the epilogue adds the two and
// multiplies by 2^(e_b + e_j - 6). hi + lo holds v to about 2^-8 relative (2^-10 absolute
// below the E4M3 normal range, 2^-18 of the row's largest value): the precision of the bf16
// operands the BF16 path multiplies. (v is rounded to fp16 on the way, 2^-11 relative; the
// residual v - hi is then exact in fp16.)
//
// The shared expert (BF16) runs in the same kernel: its stages are 64 K of bf16 weights for
// both blocks and one bf16 token slice, multiplied by kind::f16 MMAs as they land.
//
// Each stage's token slices and weight boxes land on barriers of their own, and the token
// slices are requested first: the prep warps start on a stage as soon as its token rows are
// in, while its weights are still on the way.
//
// Roles per CTA (persistent, one CTA per SM, static round-robin over tiles):
//   warp 0       producer: token slices + two weight boxes per stage
//   warp 1       MMA issuer and TMEM owner (2 accumulator buffers x 2 blocks x 64 columns)
//   warps 2..5   epilogue (TMEM lane quarter warp % 4)
//   warps 6..    token prep (kF8Prep warps): the E4M3 hi/lo B operands of routed stages
// Every wait is bounded; on expiry the CTA drains its own copies and MMAs, frees TMEM and
// returns with the device error word set.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "epilogue.cuh"

namespace moe {
namespace {

constexpr int kF8Prep = 8;                                    // token-prep warps (4 or 8)
constexpr int kF8Threads = 32 * (6 + kF8Prep);
constexpr int kF8BN = 32;                                     // token rows per chunk (decode cap)
constexpr int kF8S = 4;                                       // ring stages
constexpr uint32_t kF8WBox = 128 * 128;                       // weight box: 128 rows x 128 bytes
constexpr uint32_t kF8TokSl = kF8BN * 128;                    // bf16 token rows of a 64-wide K slice
constexpr uint32_t kF8BOp = 2 * kF8BN * 128;                  // E4M3 B operand: hi rows, then lo rows
constexpr uint32_t kF8TokOff = 2 * kF8WBox;                   // slot: weight boxes | token slices | B operands
constexpr uint32_t kF8BOff = kF8TokOff + 2 * kF8TokSl;
constexpr uint32_t kF8Slot = kF8BOff + 2 * kF8BOp;
constexpr uint32_t kF8BarOff = kF8S * kF8Slot;
constexpr uint32_t kF8NumBars = 4 * kF8S + 5;
constexpr uint32_t kF8MiscOff = kF8BarOff + 8 * kF8NumBars;
constexpr uint32_t kF8Smem = kF8MiscOff + 16 + 1024;
constexpr uint32_t kF8AccCols = 2 * kF8BN;                    // one block's accumulator (hi, lo columns)
constexpr uint32_t kF8BufCols = 2 * kF8AccCols;               // one buffer: two blocks
constexpr uint32_t kF8TmemCols = 2 * kF8BufCols;
static_assert(kF8Prep == 4 || kF8Prep == 8, "one or two prep warps per lane quarter");
static_assert(kF8Slot % 1024 == 0 && kF8BOff % 1024 == 0, "operands stay 1024-byte aligned");
static_assert(kF8Smem <= static_cast<uint32_t>(kMaxDynSmem), "ring exceeds shared memory");
static_assert(kF8TmemCols == 256, "TMEM allocation is a power of two");

struct RingF8 {
    uint64_t *wfull, *tfull;  // a stage's weight boxes / token slices landed
    uint64_t *empty, *conv, *accf, *acce, *drain;
    uint32_t *holder;
    volatile int *abort_flag;
};

__device__ __forceinline__ uint8_t *ringf8_setup(uint8_t *smem_raw, RingF8 &r)
{
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    r.wfull = reinterpret_cast<uint64_t *>(smem + kF8BarOff);
    r.tfull = r.wfull + kF8S;
    r.empty = r.tfull + kF8S;
    r.conv = r.empty + kF8S;
    r.accf = r.conv + kF8S;
    r.acce = r.accf + 2;
    r.drain = r.acce + 2;
    r.holder = reinterpret_cast<uint32_t *>(smem + kF8MiscOff);
    r.abort_flag = reinterpret_cast<volatile int *>(smem + kF8MiscOff + 4);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kF8S; ++s) {
            mbar_init(&r.wfull[s], 1);
            mbar_init(&r.tfull[s], 1);
            mbar_init(&r.empty[s], 1);
            mbar_init(&r.conv[s], kF8Prep);  // one arrival per prep warp
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
        tmem_alloc(r.holder, kF8TmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return smem;
}

// 2^n for n in [-126, 127].
__device__ __forceinline__ float pow2i(int n)
{
    return __uint_as_float(static_cast<uint32_t>(n + 127) << 23);
}

// floor(log2(v)) of a non-negative float given by its bits, clamped to [-100, 120]; 0 for
// v = 0. The clamp keeps every power of two formed from it a normal float.
__device__ __forceinline__ int exp_of(uint32_t bits)
{
    if (bits == 0u)
        return 0;
    const int e = static_cast<int>((bits >> 23) & 0xFFu) - 127;
    return e < -100 ? -100 : (e > 120 ? 120 : e);
}

// Byte offset of 16-byte chunk c of row j in a 128-byte-swizzled tile of 128-byte rows.
__device__ __forceinline__ uint32_t sw128(int j, int c)
{
    return static_cast<uint32_t>((j >> 3) * 1024 + (j & 7) * 128 + ((c ^ (j & 7)) << 4));
}

// One tile: group g (E = shared expert), chunk rows [row0, row0 + ntok), block index fb
// (128 gate/up features, or 256 down rows), K extent K.
struct TileF8 {
    int g, row0, ntok, fb, K;
    bool sh;
    __device__ __forceinline__ int npad() const { return (ntok + 15) & ~15; }
    // routed stages span one 128-wide scale block of E4M3 codes, shared stages 64 K of bf16
    __device__ __forceinline__ int stages() const { return sh ? (K + 63) / 64 : (K + 127) / 128; }
};

__device__ __forceinline__ TileF8 tile_f8(const GateUpArgs &a, int tile)
{
    int nrc, ntot;
    table_counts(a.hdr, a.max_chunks, a.err, nrc, ntot);
    TileF8 t;
    decode_gate_up<2>(a, nrc, nrc * (a.I / 128), tile, t.g, t.row0, t.ntok, t.fb);
    t.sh = t.g == a.E;
    t.K = a.H;
    return t;
}

__device__ __forceinline__ TileF8 tile_f8(const DownArgs &a, int tile)
{
    TileF8 t;
    decode_down<2>(a, tile, t.g, t.row0, t.ntok, t.fb);
    t.sh = t.g == a.E;
    t.K = t.sh ? a.Is : a.I;
    return t;
}

__device__ __forceinline__ int tiles_f8(const GateUpArgs &a)
{
    int nrc, ntot;
    table_counts(a.hdr, a.max_chunks, a.err, nrc, ntot);
    return nrc * (a.I / 128) + (ntot - nrc) * (a.Is / 128);
}

__device__ __forceinline__ int tiles_f8(const DownArgs &a)
{
    int nrc, ntot;
    table_counts(a.hdr, a.max_chunks, a.err, nrc, ntot);
    return ntot * (a.H / 256);
}

// First weight row of block b: gate_up routed rows g*2I + (b ? I : 0) + f0 of the stacked
// [E*2I, H] codes (shared: (b ? Is : 0) + f0 of [2Is, H]); down rows g*H + 256 fb + 128 b.
__device__ __forceinline__ int wrow(const GateUpArgs &a, const TileF8 &t, int b)
{
    const int f0 = t.fb * 128;
    return t.sh ? (b ? a.Is : 0) + f0 : t.g * 2 * a.I + (b ? a.I : 0) + f0;
}

__device__ __forceinline__ int wrow(const DownArgs &a, const TileF8 &t, int b)
{
    const int r = t.fb * 256 + 128 * b;
    return t.sh ? r : t.g * a.H + r;
}

// Block scales of block b of a routed tile, one per 128-wide K block: gate_up scales
// [E, 2I/128, H/128] (gate row block fb, up row block I/128 + fb), down [E, H/128, I/128]
// (row block 2 fb + b).
__device__ __forceinline__ const float *scale_row(const GateUpArgs &a, const TileF8 &t, int b)
{
    const int nbr = 2 * a.I / 128, nbc = a.H / 128;
    return a.w_scale + (static_cast<int64_t>(t.g) * nbr + (b ? a.I / 128 : 0) + t.fb) * nbc;
}

__device__ __forceinline__ const float *scale_row(const DownArgs &a, const TileF8 &t, int b)
{
    const int nbr = a.H / 128, nbc = a.I / 128;
    return a.w_scale + (static_cast<int64_t>(t.g) * nbr + 2 * t.fb + b) * nbc;
}

// e_b of a routed block: exponent of its largest scale (warp-collective).
__device__ __forceinline__ int block_exp(const float *srow, int nkb, int lane)
{
    uint32_t m = 0u;
    for (int kb = lane; kb < nkb; kb += 32)
        m = max(m, __float_as_uint(fabsf(__ldg(srow + kb))));
    return exp_of(__reduce_max_sync(0xFFFFFFFFu, m));
}

// Row maxima of the chunk's token rows: x_perm rows for gate_up, h rows for down.
__device__ __forceinline__ const uint32_t *row_amax(const GateUpArgs &a)
{
    return a.amax_in;
}

__device__ __forceinline__ const uint32_t *row_amax(const DownArgs &a)
{
    return a.amax_in;
}

// E4M3 pair (low byte = first element) of two fp16 values, saturating.
__device__ __forceinline__ uint32_t e4m3x2_of(__half2 v)
{
    return static_cast<uint32_t>(
        __nv_cvt_halfraw2_to_fp8x2(static_cast<__half2_raw>(v), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ __half2 half2_of_e4m3x2(uint32_t p)
{
    return __half2(__nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(p), __NV_E4M3));
}

// Token prep of 16 K elements: row j, K 16c .. 16c+15 of the staged bf16 token slices (two
// 64-wide slices, 128-byte swizzle) times F, split into E4M3 hi / lo and stored as chunk c of
// rows j and n + j of the B operand.
__device__ __forceinline__ void prep_chunk(const uint8_t *tok, int j, int c, float F, uint8_t *bop, int n)
{
    const uint8_t *src = tok + (c >> 2) * kF8TokSl;
    const uint4 p0 = *reinterpret_cast<const uint4 *>(src + sw128(j, 2 * (c & 3)));
    const uint4 p1 = *reinterpret_cast<const uint4 *>(src + sw128(j, 2 * (c & 3) + 1));
    const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    uint32_t hi[8], lo[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const float a0 = __uint_as_float(w[p] << 16) * F;           // K element 2p
        const float a1 = __uint_as_float(w[p] & 0xFFFF0000u) * F;   // K element 2p + 1
        const __half2 v = __floats2half2_rn(a0, a1);
        hi[p] = e4m3x2_of(v);
        lo[p] = e4m3x2_of(__hsub2(v, half2_of_e4m3x2(hi[p])));
    }
    const uint4 ho = make_uint4(hi[0] | (hi[1] << 16), hi[2] | (hi[3] << 16), hi[4] | (hi[5] << 16),
                                hi[6] | (hi[7] << 16));
    const uint4 lw = make_uint4(lo[0] | (lo[1] << 16), lo[2] | (lo[3] << 16), lo[4] | (lo[5] << 16),
                                lo[6] | (lo[7] << 16));
    *reinterpret_cast<uint4 *>(bop + sw128(j, c)) = ho;
    *reinterpret_cast<uint4 *>(bop + sw128(n + j, c)) = lw;
}

// Producer: weight boxes of block b at K element k0.
__device__ __forceinline__ void load_wbox(const GateUpArgs &a, const CUtensorMap *m, void *dst, uint64_t *bar,
                                          const TileF8 &t, int b, int k0)
{
    tma_load_2d(dst, m, bar, k0, wrow(a, t, b));
}

__device__ __forceinline__ void load_wbox(const DownArgs &a, const CUtensorMap *m, void *dst, uint64_t *bar,
                                          const TileF8 &t, int b, int k0)
{
    tma_load_2d(dst, m, bar, k0, wrow(a, t, b));
}

// gate_up epilogue of one lane quarter: g, u of features 128 fb + 32 q + lane, the chunk's
// columns; h = act(g, u) in bf16, and the largest |h| of each routed row into amax_out.
__device__ __forceinline__ void epi_f8(const GateUpArgs &a, uint32_t tb, const TileF8 &t, int q, int lane)
{
    const int64_t feat = static_cast<int64_t>(t.fb) * 128 + q * 32 + lane;
    uint16_t *out = t.sh ? a.h_sh : a.h;
    const int64_t ld = t.sh ? a.Is : a.I;
    const float L = t.sh ? a.lim_s : a.lim_r;
    const int n = t.npad();
    float ug = 1.0f, uu = 1.0f;
    if (!t.sh) {
        const int nkb = a.H / 128;
        ug = pow2i(block_exp(scale_row(a, t, 0), nkb, lane));
        uu = pow2i(block_exp(scale_row(a, t, 1), nkb, lane));
    }
    for (int c0 = 0; c0 < n; c0 += 16) {
        float gh[16], uh[16], gl[16], ul[16];
        tmem_load16(tb + c0, gh);
        tmem_load16(tb + kF8AccCols + c0, uh);
        float uj = 1.0f;  // lane i < 16: 2^(e_j - 6) of column c0 + i
        if (!t.sh) {
            tmem_load16(tb + n + c0, gl);
            tmem_load16(tb + kF8AccCols + n + c0, ul);
            if (lane < 16 && c0 + lane < t.ntok)
                uj = pow2i(exp_of(a.amax_in[t.row0 + c0 + lane]) - 6);
        }
        uint32_t mx = 0u;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float g = gh[i], u = uh[i];
            if (!t.sh) {
                const float f = __shfl_sync(0xFFFFFFFFu, uj, i);
                g = (g + gl[i]) * ug * f;
                u = (u + ul[i]) * uu * f;
            }
            const uint16_t hb = __bfloat16_as_ushort(__float2bfloat16_rn(swiglu_clip(g, u, L)));
            const int col = c0 + i;
            if (col < t.ntok)
                out[(t.row0 + col) * ld + feat] = hb;
            if (!t.sh) {
                const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, static_cast<uint32_t>(hb & 0x7FFFu));
                if (lane == i)
                    mx = m;
            }
        }
        if (!t.sh && lane < 16 && c0 + lane < t.ntok)
            atomicMax(a.amax_out + t.row0 + c0 + lane, mx << 16);
    }
}

// down epilogue of one lane quarter: output features 256 fb + 128 b + 32 q + lane of both
// blocks; routed columns add w_slot * o into y[token] (or store o_perm[slot] in the
// deterministic mode), shared columns add o.
__device__ __forceinline__ void epi_f8(const DownArgs &a, uint32_t tb, const TileF8 &t, int q, int lane)
{
    const int n = t.npad();
    float ub[2] = {1.0f, 1.0f};
    if (!t.sh) {
        const int nkb = a.I / 128;
        ub[0] = pow2i(block_exp(scale_row(a, t, 0), nkb, lane));
        ub[1] = pow2i(block_exp(scale_row(a, t, 1), nkb, lane));
    }
    for (int c0 = 0; c0 < n; c0 += 16) {
        // lane i < 16: destination row and weight (with 2^(e_j - 6)) of column c0 + i
        int64_t dst_row = -1;
        float wgt = 0.0f;
        if (lane < 16 && c0 + lane < t.ntok) {
            const int64_t rr = t.row0 + c0 + lane;
            if (!down_dst_row(a, t.sh, rr, dst_row))
                dst_row = -1;
            wgt = t.sh ? 1.0f : a.w_perm[rr] * pow2i(exp_of(a.amax_in[rr]) - 6);
        }
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const int64_t feat = static_cast<int64_t>(t.fb) * 256 + 128 * b + q * 32 + lane;
            const uint32_t tbb = tb + b * kF8AccCols;
            float oh[16], ol[16];
            tmem_load16(tbb + c0, oh);
            if (!t.sh)
                tmem_load16(tbb + n + c0, ol);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int64_t drow = __shfl_sync(0xFFFFFFFFu, dst_row, i);
                const float w = __shfl_sync(0xFFFFFFFFu, wgt, i);
                if (drow >= 0) {
                    const float o = t.sh ? oh[i] : (oh[i] + ol[i]) * ub[b];
                    float *p = a.out + drow * a.H + feat;
                    if (a.deterministic)
                        *p = w * o;
                    else
                        atomicAdd(p, w * o);
                }
            }
        }
    }
}

// Waits for the last `depth` phases of `bars` that this role armed (its own copies).
__device__ __forceinline__ void drain_f8(uint64_t *bars, int depth, int issued, const WaitCfg &wc)
{
    for (int it = issued > depth ? issued - depth : 0; it < issued; ++it)
        mbar_wait_drain(&bars[it % depth], (it / depth) & 1, wc);
}

// Both GEMMs. Maps: m_w (E4M3 codes, 128 x 128-byte boxes), m_wsh (BF16 shared weights, 64
// x 128 boxes), m_tok (routed token rows: x_perm or h), m_tok_sh (shared token rows: x or
// h_sh), token boxes of 64 K x 32 rows.
template <class Args>
__global__ void __launch_bounds__(kF8Threads, 1)
    gemm_fp8_mma_kernel(const __grid_constant__ CUtensorMap m_w, const __grid_constant__ CUtensorMap m_wsh,
                        const __grid_constant__ CUtensorMap m_tok, const __grid_constant__ CUtensorMap m_tok_sh,
                        const Args a, const WaitCfg wc)
{
    extern __shared__ uint8_t smem_raw[];
    RingF8 r;
    uint8_t *smem = ringf8_setup(smem_raw, r);
    const uint32_t tmem = *r.holder;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tiles = tiles_f8(a);

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_map(&m_w);
            tma_prefetch_map(&m_wsh);
            tma_prefetch_map(&m_tok);
            tma_prefetch_map(&m_tok_sh);
            int it = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < tiles && !stop; tile += gridDim.x) {
                const TileF8 t = tile_f8(a, tile);
                const int nst = t.stages();
                for (int st = 0; st < nst; ++st, ++it) {
                    const int s = it % kF8S;
                    if (!mbar_wait(&r.empty[s], ((it / kF8S) & 1) ^ 1, wc, r.abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *slot = smem + s * kF8Slot;
                    const int nsl = t.sh ? 1 : 2;  // 64-wide token slices of the stage
                    const int k0 = st * (t.sh ? 64 : 128);
                    mbar_arrive_expect_tx(&r.tfull[s], nsl * kF8TokSl);
                    for (int sl = 0; sl < nsl; ++sl)
                        tma_load_2d(slot + kF8TokOff + sl * kF8TokSl, t.sh ? &m_tok_sh : &m_tok, &r.tfull[s],
                                    k0 + sl * 64, t.row0);
                    mbar_arrive_expect_tx(&r.wfull[s], 2 * kF8WBox);
                    for (int b = 0; b < 2; ++b)
                        load_wbox(a, t.sh ? &m_wsh : &m_w, slot + b * kF8WBox, &r.wfull[s], t, b, k0);
                }
            }
            drain_f8(r.tfull, kF8S, it, wc);
            drain_f8(r.wfull, kF8S, it, wc);
        }
    } else if (warp == 1) {
        // MMA: routed stages multiply the E4M3 weight boxes by the hi/lo B operands (N = 2n),
        // shared stages the bf16 weight boxes by the bf16 token slice (N = n). The prep warps
        // arrive on conv after the stage's token rows landed; the weights have a barrier of
        // their own.
        if (lane == 0) {
            int it = 0, tc = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tc) {
                const TileF8 t = tile_f8(a, tile);
                const int buf = tc & 1;
                if (!mbar_wait(&r.acce[buf], ((tc >> 1) & 1) ^ 1, wc, r.abort_flag))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + buf * kF8BufCols;
                const int n = t.npad();
                const uint32_t idesc = t.sh ? idesc_bf16_f32(128, n) : idesc_e4m3_f32(128, 2 * n);
                const int nst = t.stages();
                for (int st = 0; st < nst; ++st, ++it) {
                    const int s = it % kF8S;
                    if (!mbar_wait(&r.conv[s], (it / kF8S) & 1, wc, r.abort_flag) ||
                        !mbar_wait(&r.wfull[s], (it / kF8S) & 1, wc, r.abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t slot = smem_u32(smem + s * kF8Slot);
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        const uint64_t ad = sdesc_kmajor_sw128(slot + b * kF8WBox);
                        const uint64_t bd = sdesc_kmajor_sw128(slot + (t.sh ? kF8TokOff : kF8BOff + b * kF8BOp));
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {  // 32 bytes of each 128-byte row per MMA
                            if (t.sh)
                                umma_bf16(d + b * kF8AccCols, ad + 2 * ks, bd + 2 * ks, idesc, (st | ks) != 0);
                            else
                                umma_e4m3(d + b * kF8AccCols, ad + 2 * ks, bd + 2 * ks, idesc, (st | ks) != 0);
                        }
                    }
                    umma_commit(&r.empty[s]);
                }
                if (ok)
                    umma_commit(&r.accf[buf]);
            }
            umma_commit(r.drain);
            mbar_wait_drain(r.drain, 0, wc);
        }
    } else if (warp < 6) {
        // epilogue: warps 2..5, lane quarter q
        const int q = warp & 3;
        int tc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
            const TileF8 t = tile_f8(a, tile);
            const int buf = tc & 1;
            if (!warp_wait(&r.accf[buf], (tc >> 1) & 1, wc, r.abort_flag))
                break;
            tc_fence_after();
            epi_f8(a, tmem + buf * kF8BufCols + (static_cast<uint32_t>(q * 32) << 16), t, q, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&r.acce[buf]);
        }
    } else {
        // token prep: warps 6 ..; thread p handles 16-K chunk c = p % 8 of rows j0 = (p / 8) % 16
        // and j0 + 16, for both blocks (four prep warps) or for block p / 128 (eight)
        const int p = threadIdx.x - 6 * 32;
        const int c = p & 7, j0 = (p >> 3) & 15;
        constexpr int kBlocksPer = 8 / kF8Prep;
        const int bfirst = kF8Prep == 8 ? (p >> 7) : 0;
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            const TileF8 t = tile_f8(a, tile);
            const int n = t.npad();
            const int nst = t.stages();
            // per tile: 2^-e_b of this thread's blocks, 2^(6 - e_j) of its rows (0 past the chunk)
            float pb[kBlocksPer], f0 = 0.0f, f1 = 0.0f;
            const float *sr[kBlocksPer];
            if (!t.sh) {
                const int nkb = t.K / 128;
#pragma unroll
                for (int q = 0; q < kBlocksPer; ++q) {
                    sr[q] = scale_row(a, t, bfirst + q);
                    pb[q] = pow2i(-block_exp(sr[q], nkb, lane));
                }
                const uint32_t *am = row_amax(a);
                if (j0 < t.ntok)
                    f0 = pow2i(6 - exp_of(am[t.row0 + j0]));
                if (j0 + 16 < t.ntok)
                    f1 = pow2i(6 - exp_of(am[t.row0 + j0 + 16]));
            }
            for (int st = 0; st < nst; ++st, ++it) {
                const int s = it % kF8S;
                if (!warp_wait(&r.tfull[s], (it / kF8S) & 1, wc, r.abort_flag)) {
                    ok = false;
                    break;
                }
                if (!t.sh) {
                    uint8_t *slot = smem + s * kF8Slot;
                    const uint8_t *tok = slot + kF8TokOff;
#pragma unroll
                    for (int q = 0; q < kBlocksPer; ++q) {
                        const float sb = __ldg(sr[q] + st) * pb[q];
                        uint8_t *bop = slot + kF8BOff + (bfirst + q) * kF8BOp;
                        prep_chunk(tok, j0, c, sb * f0, bop, n);
                        if (n > 16)
                            prep_chunk(tok, j0 + 16, c, sb * f1, bop, n);
                    }
                    fence_proxy_async_smem();  // the B operands are read by the tensor cores
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&r.conv[s]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kF8TmemCols);
    }
}

template <class Args>
cudaError_t launch_f8(int grid, cudaStream_t stream, const CUtensorMap &m0, const CUtensorMap &m1,
                      const CUtensorMap &m2, const CUtensorMap &m3, const Args &a, const WaitCfg &wc)
{
    constexpr int smem = static_cast<int>(kF8Smem);
    auto kernel = gemm_fp8_mma_kernel<Args>;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    kernel<<<grid, kF8Threads, smem, stream>>>(m0, m1, m2, m3, a, wc);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_up_fp8_mma(const CUtensorMap &tm_w, const CUtensorMap &tm_wsh, const CUtensorMap &tm_xp,
                                   const CUtensorMap &tm_x, const GateUpArgs &a, const WaitCfg &wc, int grid,
                                   cudaStream_t stream)
{
    return launch_f8<GateUpArgs>(grid, stream, tm_w, tm_wsh, tm_xp, tm_x, a, wc);
}

cudaError_t launch_down_fp8_mma(const CUtensorMap &tm_wd, const CUtensorMap &tm_wdsh, const CUtensorMap &tm_h,
                                const CUtensorMap &tm_hsh, const DownArgs &a, const WaitCfg &wc, int grid,
                                cudaStream_t stream)
{
    return launch_f8<DownArgs>(grid, stream, tm_wd, tm_wdsh, tm_h, tm_hsh, a, wc);
}

}  // namespace moe
