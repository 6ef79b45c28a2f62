// moe_api.cu — C ABI of the B200 MoE layer (declarations and contract in include/moe_b200.h).
//
// Host side only: argument validation (before anything is enqueued), workspace layout,
// TMA tensor-map encoding, and the launch sequence router -> permute -> gather/tile
// table -> gate_up GEMM -> down GEMM (-> combine). The library allocates nothing and never
// synchronises except in moe_check_device().
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/moe_b200.h"
#include "internal.h"

namespace {

// Device error word (bit flags of moe::kDevErr*), one per device context.
__device__ uint32_t g_moe_err;

std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};

// Optional stage events recorded by moe_forward (profiling hook).
constexpr int kMaxStageEvents = 7;
std::mutex g_ev_mu;
cudaEvent_t g_stage_ev[kMaxStageEvents];
int g_stage_n = 0;

bool stage_mark(int i, cudaStream_t s)
{
    std::lock_guard<std::mutex> lk(g_ev_mu);
    return i >= g_stage_n || cudaEventRecord(g_stage_ev[i], s) == cudaSuccess;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int num_sms = 0;
    uint32_t *err = nullptr;  // device address of g_moe_err in the current context (looked up per call)
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

moe_status_t device_info(DeviceInfo &out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return MOE_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        d.ready = true;
    }
    // The error word's address belongs to the current context's copy of this module: a
    // runtime query on every call, so no saved address outlives its context (after
    // cudaDeviceReset the module may load at another address).
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_moe_err) != cudaSuccess || p == nullptr)
        return MOE_ERR_CUDA;
    out = d;
    out.err = static_cast<uint32_t *>(p);
    return MOE_OK;
}

moe::WaitCfg wait_cfg(const DeviceInfo &d)
{
    return moe::WaitCfg{g_wait_limit_ns.load(), d.err};
}

// bf16 tensor map, 128-byte swizzle, 64-element inner box. dims/strides innermost first;
// strides (bytes) are given for dims 1..rank-1.
bool encode_bf16(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
                 const cuuint32_t *box)
{
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
                                const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// fp32 [rows, cols] row-major as the destination of 32 x 32 boxes (128 bytes wide, 128-byte
// swizzle), for tiled stores
bool map_rows_f32_store(CUtensorMap *m, const void *base, int64_t cols, int64_t rows)
{
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 4};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool map_rows(CUtensorMap *m, const void *base, int64_t cols, int64_t rows, uint32_t box_rows)
{
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {64, box_rows};
    return encode_bf16(m, base, 2, dims, strides, box);
}

// Stacked gate_up weights [G, 2*Iw, H] viewed as (H, half, row, group) so one box of
// (64, 2, feats, 1) lands as 2 * feats rows alternating gate row i / up row i.
bool map_gate_up(CUtensorMap *m, const void *base, int64_t H, int64_t Iw, int64_t G, uint32_t feats)
{
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(H), 2, static_cast<cuuint64_t>(Iw),
                                static_cast<cuuint64_t>(G)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(Iw * H * 2), static_cast<cuuint64_t>(H * 2),
                                   static_cast<cuuint64_t>(2 * Iw * H * 2)};
    const cuuint32_t box[4] = {64, 2, feats, 1};
    return encode_bf16(m, base, 4, dims, strides, box);
}

// E4M3 code tensor maps (one byte per element), inner box of `inner` = 128 bytes, 128-byte
// swizzle (converter threads read one row each without bank conflicts).
bool encode_u8(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
               const cuuint32_t *box)
{
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, static_cast<cuuint32_t>(rank),
                                const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// E4M3 gate_up codes [E, 2*Iw, H] viewed as (H, half, row, expert) like map_gate_up.
bool map_gate_up_u8(CUtensorMap *m, const void *base, int64_t H, int64_t Iw, int64_t G, uint32_t feats,
                    uint32_t inner)
{
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(H), 2, static_cast<cuuint64_t>(Iw),
                                static_cast<cuuint64_t>(G)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(Iw * H), static_cast<cuuint64_t>(H),
                                   static_cast<cuuint64_t>(2 * Iw * H)};
    const cuuint32_t box[4] = {inner, 2, feats, 1};
    return encode_u8(m, base, 4, dims, strides, box);
}

bool map_rows_u8(CUtensorMap *m, const void *base, int64_t cols, int64_t rows, uint32_t box_rows, uint32_t inner)
{
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
    const cuuint32_t box[2] = {inner, box_rows};
    return encode_u8(m, base, 2, dims, strides, box);
}

// Expert-parallel limits: ranks of one dispatch, and ranks x local experts of the per-source
// count table the receive side scans.
constexpr int kMaxEpRanks = 64;
constexpr int64_t kMaxEpTable = 8192;

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

moe_status_t check_desc(const moe_layer_desc *d)
{
    if (!d)
        return MOE_ERR_INVALID_ARG;
    if (d->T < 0 || d->H <= 0 || d->E <= 0 || d->k <= 0 || d->I <= 0 || d->Is <= 0)
        return MOE_ERR_INVALID_ARG;
    if (d->k > d->E || d->k > 32)
        return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(d->scale) || !std::isfinite(d->limit_routed) || !std::isfinite(d->limit_shared) ||
        d->limit_routed < 0.0f || d->limit_shared < 0.0f)
        return MOE_ERR_INVALID_ARG;
    if ((d->norm_expert_weight != 0 && d->norm_expert_weight != 1) ||
        (d->deterministic != 0 && d->deterministic != 1))
        return MOE_ERR_INVALID_ARG;
    if (d->E > 512 || d->H % 128 != 0 || d->I % 64 != 0 || d->Is % 64 != 0)
        return MOE_ERR_UNSUPPORTED;
    const int64_t rows = static_cast<int64_t>(d->T) * (d->k + 1);
    if (rows >= (int64_t(1) << 31) - 512 || static_cast<int64_t>(d->E) * d->H >= (int64_t(1) << 31))
        return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

struct WsLayout {
    size_t x_perm, w_perm, h, h_sh, chunks, chunks_d, hdr, o_perm, idx, w, counts, offsets, perm_token, slot_of, amax,
        total;
};

size_t up256(size_t v)
{
    return (v + 255) / 256 * 256;
}

WsLayout ws_layout(const moe_layer_desc &d)
{
    const size_t T = d.T, H = d.H, E = d.E, k = d.k, I = d.I, Is = d.Is;
    WsLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += up256(bytes);
        return o;
    };
    L.x_perm = take(T * k * H * 2);
    L.w_perm = take(T * k * 4);
    L.h = take(T * k * I * 2);
    L.h_sh = take(T * Is * 2);
    // chunk tables of gate_up and (when its cap differs) of down, sized for both weight
    // formats; the second region also holds the shared expert's two tables when FP8 routed
    // experts run with the BF16 shared expert on the pair kernels; hdr holds three headers
    const moe::GemmConfig cfg = moe::gemm_config(d.T, d.k, d.E, d.H, d.I, d.Is);
    const moe::GemmConfig cfg8 = moe::gemm_config_fp8(d.T, d.k, d.E);
    const int cap_min = cfg.cap < cfg8.cap ? cfg.cap : cfg8.cap;
    L.chunks = take(static_cast<size_t>(moe::max_chunks(d.T, d.k, d.E, cap_min)) * 16);
    L.chunks_d = take(static_cast<size_t>(moe::max_chunks(d.T, d.k, d.E, cfg.cap_d)) * 16);
    L.hdr = take(64);
    L.o_perm = take(d.deterministic ? (T * k + T) * H * 4 : 0);
    L.idx = take(T * k * 4);
    L.w = take(T * k * 4);
    L.counts = take((E + 1) * 4);
    L.offsets = take((E + 2) * 4);
    L.perm_token = take((T * k + T) * 4);
    L.slot_of = take(T * k * 4);
    // row maxima of x_perm and h (FP8 weights on the FP8 tensor cores)
    L.amax = take(T * k * 8);
    L.total = off;
    return L;
}

// Token-row maps of the pair kernels: routed rows [rows_r, cols] and shared rows [rows_s,
// cols_s] (cols_s = cols unless given), boxes of 32, 64, 96 and 128 rows.
bool pair_token_maps(moe::TokMaps *t, const void *routed, const void *shared, int64_t cols, int64_t rows_r,
                     int64_t rows_s, int64_t cols_s = 0)
{
    for (int i = 0; i < moe::kPairTokBoxes; ++i) {
        const uint32_t b = static_cast<uint32_t>(moe::kPairTokBoxStep * (i + 1));
        if (!map_rows(&t->routed_b[i], routed, cols, rows_r, b) ||
            !map_rows(&t->shared_b[i], shared, cols_s ? cols_s : cols, rows_s, b))
            return false;
    }
    return true;
}

template <typename P>
P *at(void *ws, size_t off)
{
    return reinterpret_cast<P *>(static_cast<uint8_t *>(ws) + off);
}

moe_status_t cuda_status(cudaError_t e)
{
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t run_router(const moe_layer_desc &d, const DeviceInfo &di, const uint16_t *x, const uint16_t *Wr,
                        const float *bias, int32_t *idx, float *w, float *margin, cudaStream_t s)
{
    CUtensorMap tm_x, tm_wr;
    const moe::RouterSplit sp = moe::router_split(d.E, d.T, d.H, di.num_sms);
    if (!map_rows(&tm_x, x, d.H, d.T, 128) || !map_rows(&tm_wr, Wr, d.H, d.E, sp.box_rows))
        return MOE_ERR_CUDA;
    moe::RouterArgs a{bias, idx, w, margin, d.T, d.H, d.E, d.k, d.scale, d.norm_expert_weight, di.num_sms};
    return cuda_status(moe::launch_router(tm_x, tm_wr, a, wait_cfg(di), s));
}

// Expert weights of one call: BF16 routed experts, or FP8 E4M3 codes with 128x128 block
// scales (gu_scale / d_scale non-NULL); the shared expert is BF16 in both.
struct ExpertWeights {
    const void *gu, *d;
    const float *gu_scale, *d_scale;
    const uint16_t *sh_gu, *sh_d;
    bool fp8() const { return gu_scale != nullptr; }
};

// Which expert groups one call computes: the layer (routed + shared), the routed experts of
// dispatched rows only (expert parallelism's owner side), or the shared expert only.
enum class FfnGroups { kBoth, kRoutedOnly, kSharedOnly };

moe_status_t run_expert_ffn(const moe_layer_desc &d, const DeviceInfo &di, const uint16_t *x, const float *topk_w,
                            const int32_t *offsets, const int32_t *perm_token, const int32_t *slot_of,
                            const ExpertWeights &Win, float *out, void *ws, cudaStream_t s,
                            FfnGroups groups = FfnGroups::kBoth)
{
    // a group that is not computed has no tiles; its tensor maps only need a valid address
    ExpertWeights W = Win;
    if (groups == FfnGroups::kRoutedOnly) {
        W.sh_gu = static_cast<const uint16_t *>(W.gu);
        W.sh_d = static_cast<const uint16_t *>(W.d);
    } else if (groups == FfnGroups::kSharedOnly) {
        W.gu = W.sh_gu;
        W.d = W.sh_d;
    }
    const bool fp8 = W.fp8();
    const WsLayout L = ws_layout(d);
    uint16_t *x_perm = at<uint16_t>(ws, L.x_perm);
    float *w_perm = at<float>(ws, L.w_perm);
    uint16_t *h = at<uint16_t>(ws, L.h);
    uint16_t *h_sh = at<uint16_t>(ws, L.h_sh);
    const moe::GemmConfig cfg = fp8 ? moe::gemm_config_fp8(d.T, d.k, d.E) : moe::gemm_config(d.T, d.k, d.E, d.H, d.I, d.Is);
    int4 *chunks = at<int4>(ws, L.chunks);
    int32_t *hdr = at<int32_t>(ws, L.hdr);
    // down reads the gate_up table unless its cap differs
    int4 *chunks_d = cfg.cap_d != cfg.cap ? at<int4>(ws, L.chunks_d) : chunks;
    int32_t *hdr_d = cfg.cap_d != cfg.cap ? hdr + 4 : hdr;
    const int64_t Tk = static_cast<int64_t>(d.T) * d.k;

    // One TMA box per weight operand and pipeline stage: all weight tiles of a stage (64 * mt
    // gate/up feature pairs, or 128 * mt_d down rows). Token rows come in one box of the
    // chunk cap on single CTAs, in one 64- or 128-row box per K slice on CTA pairs.
    const uint32_t brows = static_cast<uint32_t>(cfg.cap);
    const uint32_t feats = static_cast<uint32_t>(64 * cfg.mt);
    const uint32_t drows = static_cast<uint32_t>(128 * cfg.mt_d);
    CUtensorMap tm_w, tm_wsh, tm_wd, tm_wdsh;
    moe::TokMaps tok_gu, tok_d;  // token rows of gate_up (x_perm, x) and down (h, h_sh)
    const int64_t EH = static_cast<int64_t>(d.E) * d.H;
    const uint32_t inner8 = 128;  // one 128-wide scale block of E4M3 codes per stage
    // FP8 decode on the FP8 tensor cores: weights as plain row-major boxes of 128 rows (E4M3
    // codes 128 bytes wide, the BF16 shared expert 64 elements wide)
    const bool f8mma = fp8 && moe::fp8_mma_config(cfg, d.H, d.I, d.Is);
    bool ok = map_rows(&tok_gu.routed, x_perm, d.H, Tk, brows) && map_rows(&tok_gu.shared, x, d.H, d.T, brows) &&
              map_rows(&tok_d.routed, h, d.I, Tk, brows) && map_rows(&tok_d.shared, h_sh, d.Is, d.T, brows);
    if (ok && f8mma)
        ok = map_rows_u8(&tm_w, W.gu, d.H, static_cast<int64_t>(d.E) * 2 * d.I, 128, inner8) &&
             map_rows_u8(&tm_wd, W.d, d.I, EH, 128, inner8) && map_rows(&tm_wsh, W.sh_gu, d.H, 2 * d.Is, 128) &&
             map_rows(&tm_wdsh, W.sh_d, d.Is, d.H, 128);
    else if (ok)
        ok = (fp8 ? map_gate_up_u8(&tm_w, W.gu, d.H, d.I, d.E, feats, inner8)
                  : map_gate_up(&tm_w, W.gu, d.H, d.I, d.E, feats)) &&
             (fp8 ? map_rows_u8(&tm_wd, W.d, d.I, EH, drows, inner8) : map_rows(&tm_wd, W.d, d.I, EH, drows)) &&
             map_gate_up(&tm_wsh, W.sh_gu, d.H, d.Is, 1, feats) && map_rows(&tm_wdsh, W.sh_d, d.Is, d.H, drows);
    uint32_t *amax_x = f8mma ? at<uint32_t>(ws, L.amax) : nullptr;
    uint32_t *amax_h = f8mma ? amax_x + Tk : nullptr;
    if (ok && cfg.pair)
        ok = pair_token_maps(&tok_gu, x_perm, x, d.H, Tk, d.T) && pair_token_maps(&tok_d, h, h_sh, d.I, Tk, d.T, d.Is);
    if (!ok)
        return MOE_ERR_CUDA;

    // FP8 prefill: the routed experts run on the FP8 kernels and the BF16 shared expert on
    // the BF16 CTA-pair kernels (full 128-wide K stages, no conversion), as a group of its
    // own (expert count 0, so its chunks are the shared group) with tile tables in the
    // second table region, which the FP8 configuration leaves unused (one table, cap ==
    // cap_d), and headers at hdr + 4 / hdr + 8.
    const moe::GemmConfig cfg_sh = moe::gemm_config(d.T, d.k, d.E, d.H, d.I, d.Is);
    const bool split = fp8 && groups == FfnGroups::kBoth && cfg.cap > 32 && cfg_sh.pair;
    CUtensorMap tm_wsh2, tm_wdsh2;
    moe::TokMaps tok_gu2, tok_d2;  // the shared expert's token rows as routed-position maps
    int4 *chunks_s = nullptr, *chunks_sd = nullptr;
    if (split) {
        const int64_t n_gu = (d.T + cfg_sh.cap - 1) / cfg_sh.cap + 1;
        const int64_t n_d = (d.T + cfg_sh.cap_d - 1) / cfg_sh.cap_d + 1;
        if (n_gu + n_d > moe::max_chunks(d.T, d.k, d.E, cfg_sh.cap_d))
            return MOE_ERR_WORKSPACE;
        chunks_s = at<int4>(ws, L.chunks_d);
        chunks_sd = chunks_s + n_gu;
        // the shared expert runs as the only group: its rows are the "shared" maps
        if (!(map_gate_up(&tm_wsh2, W.sh_gu, d.H, d.Is, 1, static_cast<uint32_t>(64 * cfg_sh.mt)) &&
              map_rows(&tm_wdsh2, W.sh_d, d.Is, d.H, static_cast<uint32_t>(128 * cfg_sh.mt_d)) &&
              pair_token_maps(&tok_gu2, x, x, d.H, d.T, d.T) && pair_token_maps(&tok_d2, h_sh, h_sh, d.Is, d.T, d.T)))
            return MOE_ERR_CUDA;
    }

    if (!stage_mark(2, s))
        return MOE_ERR_CUDA;
    cudaError_t e = cudaSuccess;
    // the gather also zeroes y (the down GEMM's reduction target) when it runs
    const bool zero_in_gather = groups != FfnGroups::kSharedOnly && !d.deterministic;
    if (groups != FfnGroups::kSharedOnly)
        e = moe::launch_gather(x, topk_w, slot_of, d.T, d.k, d.H, x_perm, w_perm, di.num_sms, di.err, s,
                               zero_in_gather ? out : nullptr, amax_x, amax_h);
    const int shared_rows = groups == FfnGroups::kRoutedOnly || split ? 0 : d.T;
    const int nch = static_cast<int>(moe::max_chunks(d.T, d.k, d.E, cfg.cap));
    const int nch_d = static_cast<int>(moe::max_chunks(d.T, d.k, d.E, cfg.cap_d));
    int nch_s = 0, nch_sd = 0;  // shared-expert tables of the FP8 split (see above)
    if (split) {
        nch_s = static_cast<int>(chunks_sd - chunks_s);
        nch_sd = static_cast<int>(moe::max_chunks(d.T, d.k, d.E, cfg_sh.cap_d)) - nch_s;
    }
    if (e == cudaSuccess)
        e = moe::launch_chunks(offsets, d.E, shared_rows, cfg.cap, chunks, hdr, cfg.cap_d,
                               cfg.cap_d != cfg.cap ? chunks_d : nullptr, hdr_d, nch, nch_d, Tk, di.err, s);
    if (e == cudaSuccess && split)
        e = moe::launch_chunks(offsets, 0, d.T, cfg_sh.cap, chunks_s, hdr + 4, cfg_sh.cap_d, chunks_sd, hdr + 8,
                               nch_s, nch_sd, Tk, di.err, s);
    if (e == cudaSuccess && !d.deterministic && !zero_in_gather)
        e = cudaMemsetAsync(out, 0, static_cast<size_t>(d.T) * d.H * 4, s);
    if (e != cudaSuccess)
        return MOE_ERR_CUDA;
    const moe::WaitCfg wc = wait_cfg(di);
    moe::GateUpArgs ga{chunks, hdr, h, h_sh, d.E, d.H, d.I, d.Is, d.limit_routed, d.limit_shared, W.gu_scale,
                       Tk, d.T, nch, cfg.cap, di.err, amax_x, amax_h};
    if (!stage_mark(3, s))
        return MOE_ERR_CUDA;
    if (f8mma)
        e = moe::launch_gate_up_fp8_mma(tm_w, tm_wsh, tok_gu.routed, tok_gu.shared, ga, wc, di.num_sms, s);
    else
        e = fp8 ? moe::launch_gate_up_fp8(tm_w, tm_wsh, tok_gu.routed, tok_gu.shared, ga, wc, di.num_sms, cfg, s)
                : moe::launch_gate_up(tm_w, tm_wsh, tok_gu, ga, wc, di.num_sms, cfg, s);
    if (e == cudaSuccess && split) {
        const moe::GateUpArgs gs{chunks_s, hdr + 4, h, h_sh, 0, d.H, d.I, d.Is, d.limit_routed, d.limit_shared,
                                 nullptr, Tk, d.T, nch_s, cfg_sh.cap, di.err};
        e = moe::launch_gate_up(tm_wsh2, tm_wsh2, tok_gu2, gs, wc, di.num_sms, cfg_sh, s);
    }
    if (e != cudaSuccess)
        return MOE_ERR_CUDA;
    moe::DownArgs da{chunks_d, hdr_d, perm_token, w_perm, out, d.E, d.H, d.I, d.Is, d.T, d.k, d.deterministic,
                     W.d_scale, cfg.cap_d != cfg.cap ? nch_d : nch, cfg.cap_d, di.err, amax_h};
    if (!stage_mark(4, s))
        return MOE_ERR_CUDA;
    if (f8mma)
        e = moe::launch_down_fp8_mma(tm_wd, tm_wdsh, tok_d.routed, tok_d.shared, da, wc, di.num_sms, s);
    else
        e = fp8 ? moe::launch_down_fp8(tm_wd, tm_wdsh, tok_d.routed, tok_d.shared, da, wc, di.num_sms, cfg, s)
                : moe::launch_down(tm_wd, tm_wdsh, tok_d, da, wc, di.num_sms, cfg, s);
    if (e == cudaSuccess && split) {
        const moe::DownArgs ds{chunks_sd, hdr + 8, perm_token, w_perm, out, 0, d.H, d.I, d.Is, d.T, d.k,
                               d.deterministic, nullptr, nch_sd, cfg_sh.cap_d, di.err};
        e = moe::launch_down(tm_wdsh2, tm_wdsh2, tok_d2, ds, wc, di.num_sms, cfg_sh, s);
    }
    if (e != cudaSuccess || !stage_mark(5, s))
        return MOE_ERR_CUDA;
    return MOE_OK;
}

// Everything after routing: permutation -> expert FFNs (-> fixed-order combine).
moe_status_t forward_routed(const moe_layer_desc &d, const DeviceInfo &di, const uint16_t *x, const int32_t *idx,
                            const float *w, const ExpertWeights &W, float *y, void *ws, cudaStream_t s)
{
    const WsLayout L = ws_layout(d);
    int32_t *counts = at<int32_t>(ws, L.counts);
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *perm_token = at<int32_t>(ws, L.perm_token);
    int32_t *slot_of = at<int32_t>(ws, L.slot_of);
    if (!stage_mark(1, s))
        return MOE_ERR_CUDA;
    const moe::PermuteArgs pa{idx, d.T, d.k, d.E, counts, offsets, perm_token, slot_of, nullptr, nullptr, nullptr,
                              nullptr, 0, di.err, 0};
    if (moe::launch_permute(pa, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    float *out = d.deterministic ? at<float>(ws, L.o_perm) : y;
    moe_status_t st = run_expert_ffn(d, di, x, w, offsets, perm_token, slot_of, W, out, ws, s);
    if (st != MOE_OK)
        return st;
    if (d.deterministic) {
        st = cuda_status(moe::launch_combine(out, slot_of, d.T, d.k, d.H, y, di.err, s));
        if (st == MOE_OK && !stage_mark(6, s))
            st = MOE_ERR_CUDA;
    }
    return st;
}

// ---------------------------------------------------------------- backward
struct BwdLayout {
    size_t counts, offsets, perm_token, slot_of, poff, chunks, wgroups, hdr, x_pad, dy_pad, w_pad, tok_pad, gu_r,
        gu_s, dgu_r, dgu_s, hw_r, hw_s, dw_pad, dl_pad, total;
    int64_t P_s, P_r_max, P_max;
};

// Sizes are upper bounds: each routed group pads fewer than 64 rows.
BwdLayout bwd_layout(const moe_layer_desc &d)
{
    const size_t T = d.T, H = d.H, E = d.E, k = d.k, I = d.I, Is = d.Is;
    BwdLayout L{};
    L.P_s = (static_cast<int64_t>(T) + moe::kBwdPad - 1) / moe::kBwdPad * moe::kBwdPad;
    L.P_r_max = static_cast<int64_t>(T * k + moe::kBwdPad * E);
    L.P_max = L.P_s + L.P_r_max;
    const size_t P = L.P_max, Pr = L.P_r_max, Ps = L.P_s;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += up256(bytes);
        return o;
    };
    L.counts = take((E + 1) * 4);
    L.offsets = take((E + 2) * 4);
    L.perm_token = take((T * k + T) * 4);
    L.slot_of = take(T * k * 4);
    L.poff = take((E + 2) * 4);
    L.chunks = take(((T * k + T) / moe::kBwdCap + E + 2) * 16);
    L.wgroups = take((E + 1) * 16);
    L.hdr = take(64);
    L.x_pad = take(P * H * 2);
    L.dy_pad = take(P * H * 2);
    L.w_pad = take(P * 4);
    L.tok_pad = take(P * 4);
    L.gu_r = take(Pr * 2 * I * 4);
    L.gu_s = take(Ps * 2 * Is * 4);
    L.dgu_r = take(Pr * 2 * I * 2);
    L.dgu_s = take(Ps * 2 * Is * 2);
    L.hw_r = take(Pr * I * 2);
    L.hw_s = take(Ps * Is * 2);
    L.dw_pad = take(P * 4);
    L.dl_pad = take(P * 4);
    L.total = off;
    return L;
}

moe_status_t check_bwd_desc(const moe_layer_desc *d)
{
    const moe_status_t st = check_desc(d);
    if (st != MOE_OK)
        return st;
    if (d->I % 128 != 0 || d->Is % 128 != 0)
        return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // namespace

extern "C" {

const char *moe_status_string(int status)
{
    switch (status) {
    case MOE_OK:
        return "ok";
    case MOE_ERR_INVALID_ARG:
        return "invalid argument";
    case MOE_ERR_UNSUPPORTED:
        return "unsupported shape or alignment";
    case MOE_ERR_WORKSPACE:
        return "workspace too small";
    case MOE_ERR_CUDA:
        return "CUDA error";
    case MOE_ERR_TIMEOUT:
        return "device wait timed out";
    case MOE_ERR_DEVICE_BOUNDS:
        return "device range check failed (debug build)";
    default:
        return "unknown status";
    }
}

moe_status_t moe_workspace_size(const moe_layer_desc *desc, size_t *bytes)
{
    if (!bytes)
        return MOE_ERR_INVALID_ARG;
    const moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    *bytes = ws_layout(*desc).total;
    return MOE_OK;
}

moe_status_t moe_router(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wr, const float *bias,
                        int32_t *topk_idx, float *topk_w, float *margin, void *stream)
{
    moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    if (desc->T == 0)
        return MOE_OK;  // nothing to do; array pointers may be NULL
    if (!x || !Wr || !bias || !topk_idx || !topk_w)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Wr))
        return MOE_ERR_UNSUPPORTED;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK)
        return st;
    return run_router(*desc, di, x, Wr, bias, topk_idx, topk_w, margin, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_permute(const moe_layer_desc *desc, const int32_t *topk_idx, int32_t *counts, int32_t *offsets,
                         int32_t *perm_token, int32_t *slot_of, void *stream)
{
    moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    if (desc->T == 0)
        return MOE_OK;  // nothing to do; array pointers may be NULL
    if (!topk_idx || !counts || !offsets || !perm_token || !slot_of)
        return MOE_ERR_INVALID_ARG;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK)
        return st;
    const moe::PermuteArgs pa{topk_idx, desc->T, desc->k, desc->E, counts, offsets, perm_token, slot_of,
                              nullptr, nullptr, nullptr, nullptr, 0, di.err, 0};
    return cuda_status(moe::launch_permute(pa, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_ffn(const moe_layer_desc *desc, const uint16_t *x, const float *topk_w,
                            const int32_t *offsets, const int32_t *perm_token, const int32_t *slot_of,
                            const uint16_t *W_gate_up, const uint16_t *W_down, const uint16_t *Wsh_gate_up,
                            const uint16_t *Wsh_down, float *out, void *ws, size_t ws_bytes, void *stream)
{
    moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    if (desc->T == 0)
        return MOE_OK;  // nothing to do; array pointers may be NULL
    if (!x || !topk_w || !offsets || !perm_token || !slot_of || !W_gate_up || !W_down || !Wsh_gate_up ||
        !Wsh_down || !out || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W_gate_up) || !aligned16(W_down) || !aligned16(Wsh_gate_up) ||
        !aligned16(Wsh_down) || !aligned16(out) || !aligned16(ws))
        return MOE_ERR_UNSUPPORTED;
    if (ws_bytes < ws_layout(*desc).total)
        return MOE_ERR_WORKSPACE;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK)
        return st;
    const ExpertWeights W{W_gate_up, W_down, nullptr, nullptr, Wsh_gate_up, Wsh_down};
    return run_expert_ffn(*desc, di, x, topk_w, offsets, perm_token, slot_of, W, out, ws,
                          static_cast<cudaStream_t>(stream));
}

moe_status_t moe_combine(const moe_layer_desc *desc, const float *o_perm, const int32_t *slot_of, float *y,
                         void *stream)
{
    moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    if (desc->T == 0)
        return MOE_OK;  // nothing to do; array pointers may be NULL
    if (!o_perm || !slot_of || !y)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(o_perm) || !aligned16(y))
        return MOE_ERR_UNSUPPORTED;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK)
        return st;
    return cuda_status(moe::launch_combine(o_perm, slot_of, desc->T, desc->k, desc->H, y, di.err,
                                           static_cast<cudaStream_t>(stream)));
}

// Device staging of moe_forward_host after the forward workspace: two input buffers
// [T, H] bf16 and two output buffers [T, H] fp32, each 256-byte aligned.
struct HostLayout {
    size_t fwd, x0, x1, y0, y1, total;
};

HostLayout host_layout(const moe_layer_desc &d)
{
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    const size_t xb = up(static_cast<size_t>(d.T) * d.H * 2), yb = up(static_cast<size_t>(d.T) * d.H * 4);
    HostLayout L;
    L.fwd = 0;
    L.x0 = up(ws_layout(d).total);
    L.x1 = L.x0 + xb;
    L.y0 = L.x1 + xb;
    L.y1 = L.y0 + yb;
    L.total = L.y1 + yb;
    return L;
}

moe_status_t moe_host_workspace_size(const moe_layer_desc *desc, size_t *bytes)
{
    if (!bytes)
        return MOE_ERR_INVALID_ARG;
    const moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    *bytes = host_layout(*desc).total;
    return MOE_OK;
}

moe_status_t moe_forward_host(const moe_layer_desc *desc, int32_t n_batches, const uint16_t *x_host,
                              const uint16_t *Wr, const float *bias, const void *W_gate_up, const float *W_gate_up_scale,
                              const void *W_down, const float *W_down_scale, const uint16_t *Wsh_gate_up,
                              const uint16_t *Wsh_down, float *y_host, void *ws, size_t ws_bytes, void *stream)
{
    moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    const bool fp8 = W_gate_up_scale != nullptr;
    if (n_batches < 0 || fp8 != (W_down_scale != nullptr))
        return MOE_ERR_INVALID_ARG;
    if (desc->T == 0 || n_batches == 0)
        return MOE_OK;  // nothing to do; array pointers may be NULL
    if (!x_host || !y_host || !Wr || !bias || !W_gate_up || !W_down || !Wsh_gate_up || !Wsh_down || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(ws))
        return MOE_ERR_UNSUPPORTED;
    const HostLayout L = host_layout(*desc);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t xe = static_cast<size_t>(desc->T) * desc->H;  // elements of one batch
    uint16_t *xd[2] = {at<uint16_t>(ws, L.x0), at<uint16_t>(ws, L.x1)};
    float *yd[2] = {at<float>(ws, L.y0), at<float>(ws, L.y1)};

    // copy streams and the events that order them against the compute stream s; streams and
    // events are released by the runtime once their pending work completes. The output copy
    // of a batch is split in two halves on two streams: one device-to-host copy ran at ~44 GB/s
    // on a B200, two concurrent halves at ~57 GB/s (host-to-device: ~55 GB/s either way).
    cudaStream_t h2d = nullptr, d2h[2] = {nullptr, nullptr};
    cudaEvent_t ev[9] = {};  // start, h2d done x2, compute done x2, d2h done x2 per half
    bool ok = cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&d2h[0], cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&d2h[1], cudaStreamNonBlocking) == cudaSuccess;
    for (int i = 0; ok && i < 9; ++i)
        ok = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) == cudaSuccess;
    cudaEvent_t ev_start = ev[0], *ev_in = ev + 1, *ev_comp = ev + 3, *ev_out = ev + 5;  // ev_out[2 * b + half]
    // the copies start after the work already queued on s
    ok = ok && cudaEventRecord(ev_start, s) == cudaSuccess && cudaStreamWaitEvent(h2d, ev_start, 0) == cudaSuccess &&
         cudaStreamWaitEvent(d2h[0], ev_start, 0) == cudaSuccess &&
         cudaStreamWaitEvent(d2h[1], ev_start, 0) == cudaSuccess;
    const size_t rows0 = static_cast<size_t>(desc->T) / 2;  // rows of the first output half
    st = ok ? MOE_OK : MOE_ERR_CUDA;
    for (int i = 0; st == MOE_OK && i < n_batches; ++i) {
        const int b = i & 1;
        // input buffer b was last read by batch i - 2's forward; output buffer b last copied
        // out by batch i - 2's transfer
        if (i >= 2 && (cudaStreamWaitEvent(h2d, ev_comp[b], 0) != cudaSuccess ||
                       cudaStreamWaitEvent(s, ev_out[2 * b], 0) != cudaSuccess ||
                       cudaStreamWaitEvent(s, ev_out[2 * b + 1], 0) != cudaSuccess)) {
            st = MOE_ERR_CUDA;
            break;
        }
        if (cudaMemcpyAsync(xd[b], x_host + static_cast<size_t>(i) * xe, xe * 2, cudaMemcpyHostToDevice, h2d) !=
                cudaSuccess ||
            cudaEventRecord(ev_in[b], h2d) != cudaSuccess || cudaStreamWaitEvent(s, ev_in[b], 0) != cudaSuccess) {
            st = MOE_ERR_CUDA;
            break;
        }
        st = fp8 ? moe_forward_fp8(desc, xd[b], Wr, bias, static_cast<const uint8_t *>(W_gate_up), W_gate_up_scale,
                                   static_cast<const uint8_t *>(W_down), W_down_scale, Wsh_gate_up, Wsh_down, yd[b],
                                   nullptr, nullptr, ws, L.x0, stream)
                 : moe_forward(desc, xd[b], Wr, bias, static_cast<const uint16_t *>(W_gate_up),
                               static_cast<const uint16_t *>(W_down), Wsh_gate_up, Wsh_down, yd[b], nullptr, nullptr,
                               ws, L.x0, stream);
        if (st != MOE_OK)
            break;
        if (cudaEventRecord(ev_comp[b], s) != cudaSuccess) {
            st = MOE_ERR_CUDA;
            break;
        }
        for (int hf = 0; hf < 2 && st == MOE_OK; ++hf) {
            const size_t r0 = hf ? rows0 : 0, nr = hf ? desc->T - rows0 : rows0;
            const size_t off = static_cast<size_t>(i) * xe + r0 * desc->H;
            if (nr > 0 && (cudaStreamWaitEvent(d2h[hf], ev_comp[b], 0) != cudaSuccess ||
                           cudaMemcpyAsync(y_host + off, yd[b] + r0 * desc->H, nr * desc->H * 4,
                                           cudaMemcpyDeviceToHost, d2h[hf]) != cudaSuccess))
                st = MOE_ERR_CUDA;
            if (st == MOE_OK && cudaEventRecord(ev_out[2 * b + hf], d2h[hf]) != cudaSuccess)
                st = MOE_ERR_CUDA;
        }
    }
    // s completes after every transfer issued above (the copy streams are in order)
    for (int hf = 0; hf < 2; ++hf)
        if (d2h[hf] && ev[0] && cudaEventRecord(ev_out[hf], d2h[hf]) == cudaSuccess)
            cudaStreamWaitEvent(s, ev_out[hf], 0);
    if (h2d && ev[0] && cudaEventRecord(ev_in[0], h2d) == cudaSuccess)
        cudaStreamWaitEvent(s, ev_in[0], 0);
    for (cudaEvent_t e : ev)
        if (e)
            cudaEventDestroy(e);
    if (h2d)
        cudaStreamDestroy(h2d);
    for (cudaStream_t d : d2h)
        if (d)
            cudaStreamDestroy(d);
    return st;
}

moe_status_t moe_ep_pack(const moe_layer_desc *desc, const uint16_t *x, const float *topk_w, const int32_t *slot_of,
                         uint16_t *x_send, float *w_send, void *stream)
{
    moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    if (desc->T == 0)
        return MOE_OK;  // nothing to do; array pointers may be NULL
    if (!x || !topk_w || !slot_of || !x_send || !w_send)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_send))
        return MOE_ERR_UNSUPPORTED;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK)
        return st;
    return cuda_status(moe::launch_gather(x, topk_w, slot_of, desc->T, desc->k, desc->H, x_send, w_send, di.num_sms,
                                          di.err, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_experts(const moe_layer_desc *desc, int32_t ep_ranks, const int32_t *recv_counts,
                            const uint16_t *x_recv, const float *w_recv, const uint16_t *W_gate_up,
                            const uint16_t *W_down, float *out, void *ws, size_t ws_bytes, void *stream)
{
    moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    if (desc->k != 1 || ep_ranks < 1 || ep_ranks > kMaxEpRanks)
        return MOE_ERR_INVALID_ARG;
    if (static_cast<int64_t>(ep_ranks) * desc->E > kMaxEpTable)
        return MOE_ERR_UNSUPPORTED;
    if (desc->T == 0)
        return MOE_OK;  // nothing received; array pointers may be NULL
    if (!recv_counts || !x_recv || !w_recv || !W_gate_up || !W_down || !out || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_recv) || !aligned16(W_gate_up) || !aligned16(W_down) || !aligned16(out) || !aligned16(ws))
        return MOE_ERR_UNSUPPORTED;
    moe_layer_desc d = *desc;
    d.deterministic = 0;  // one contribution per output row: the sum order is fixed anyway
    const WsLayout L = ws_layout(d);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK)
        return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *perm_token = at<int32_t>(ws, L.perm_token);
    int32_t *slot_of = at<int32_t>(ws, L.slot_of);
    st = cuda_status(moe::launch_ep_regroup(recv_counts, ep_ranks, d.E, d.T, offsets, perm_token, slot_of, di.num_sms, s));
    if (st != MOE_OK)
        return st;
    const ExpertWeights W{W_gate_up, W_down, nullptr, nullptr, nullptr, nullptr};
    return run_expert_ffn(d, di, x_recv, w_recv, offsets, perm_token, slot_of, W, out, ws, s, FfnGroups::kRoutedOnly);
}

moe_status_t moe_shared_expert(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wsh_gate_up,
                               const uint16_t *Wsh_down, float *out, void *ws, size_t ws_bytes, void *stream)
{
    moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    if (desc->T == 0)
        return MOE_OK;  // nothing to do; array pointers may be NULL
    if (!x || !Wsh_gate_up || !Wsh_down || !out || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Wsh_gate_up) || !aligned16(Wsh_down) || !aligned16(out) || !aligned16(ws))
        return MOE_ERR_UNSUPPORTED;
    moe_layer_desc d = *desc;
    d.deterministic = 0;  // one contribution per output row
    const WsLayout L = ws_layout(d);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK)
        return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t *offsets = at<int32_t>(ws, L.offsets);  // no routed rows: every routed group is empty
    if (cudaMemsetAsync(offsets, 0, static_cast<size_t>(d.E + 2) * 4, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    const ExpertWeights W{nullptr, nullptr, nullptr, nullptr, Wsh_gate_up, Wsh_down};
    return run_expert_ffn(d, di, x, nullptr, offsets, at<int32_t>(ws, L.perm_token), at<int32_t>(ws, L.slot_of), W,
                          out, ws, s, FfnGroups::kSharedOnly);
}

moe_status_t moe_forward(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wr, const float *bias,
                         const uint16_t *W_gate_up, const uint16_t *W_down, const uint16_t *Wsh_gate_up,
                         const uint16_t *Wsh_down, float *y, int32_t *topk_idx_out, float *topk_w_out, void *ws,
                         size_t ws_bytes, void *stream)
{
    moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    if (desc->T == 0)
        return MOE_OK;  // nothing to do; array pointers may be NULL
    if (!x || !Wr || !bias || !W_gate_up || !W_down || !Wsh_gate_up || !Wsh_down || !y || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Wr) || !aligned16(W_gate_up) || !aligned16(W_down) ||
        !aligned16(Wsh_gate_up) || !aligned16(Wsh_down) || !aligned16(y) || !aligned16(ws))
        return MOE_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(*desc);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK)
        return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t *idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.idx);
    float *w = topk_w_out ? topk_w_out : at<float>(ws, L.w);
    if (!stage_mark(0, s))
        return MOE_ERR_CUDA;
    if ((st = run_router(*desc, di, x, Wr, bias, idx, w, nullptr, s)) != MOE_OK)
        return st;
    const ExpertWeights W{W_gate_up, W_down, nullptr, nullptr, Wsh_gate_up, Wsh_down};
    return forward_routed(*desc, di, x, idx, w, W, y, ws, s);
}

moe_status_t moe_forward_with_ids(const moe_layer_desc *desc, const uint16_t *x, const int32_t *topk_idx,
                                  const float *topk_w, const uint16_t *W_gate_up, const uint16_t *W_down,
                                  const uint16_t *Wsh_gate_up, const uint16_t *Wsh_down, float *y, void *ws,
                                  size_t ws_bytes, void *stream)
{
    moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    if (desc->T == 0)
        return MOE_OK;
    if (!x || !topk_idx || !topk_w || !W_gate_up || !W_down || !Wsh_gate_up || !Wsh_down || !y || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W_gate_up) || !aligned16(W_down) || !aligned16(Wsh_gate_up) ||
        !aligned16(Wsh_down) || !aligned16(y) || !aligned16(ws))
        return MOE_ERR_UNSUPPORTED;
    if (ws_bytes < ws_layout(*desc).total)
        return MOE_ERR_WORKSPACE;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK)
        return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!stage_mark(0, s))
        return MOE_ERR_CUDA;
    const ExpertWeights W{W_gate_up, W_down, nullptr, nullptr, Wsh_gate_up, Wsh_down};
    return forward_routed(*desc, di, x, topk_idx, topk_w, W, y, ws, s);
}

moe_status_t moe_forward_fp8(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wr, const float *bias,
                             const uint8_t *W_gate_up_q, const float *W_gate_up_scale, const uint8_t *W_down_q,
                             const float *W_down_scale, const uint16_t *Wsh_gate_up, const uint16_t *Wsh_down,
                             float *y, int32_t *topk_idx_out, float *topk_w_out, void *ws, size_t ws_bytes,
                             void *stream)
{
    moe_status_t st = check_desc(desc);
    if (st != MOE_OK)
        return st;
    if (desc->I % 128 != 0)
        return MOE_ERR_UNSUPPORTED;  // gate and up rows must start 128-row scale blocks
    if (desc->T == 0)
        return MOE_OK;  // nothing to do; array pointers may be NULL
    if (!x || !Wr || !bias || !W_gate_up_q || !W_gate_up_scale || !W_down_q || !W_down_scale || !Wsh_gate_up ||
        !Wsh_down || !y || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Wr) || !aligned16(W_gate_up_q) || !aligned16(W_down_q) ||
        !aligned16(Wsh_gate_up) || !aligned16(Wsh_down) || !aligned16(y) || !aligned16(ws) ||
        (reinterpret_cast<uintptr_t>(W_gate_up_scale) & 3u) || (reinterpret_cast<uintptr_t>(W_down_scale) & 3u))
        return MOE_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(*desc);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK)
        return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t *idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.idx);
    float *w = topk_w_out ? topk_w_out : at<float>(ws, L.w);
    if (!stage_mark(0, s))
        return MOE_ERR_CUDA;
    if ((st = run_router(*desc, di, x, Wr, bias, idx, w, nullptr, s)) != MOE_OK)
        return st;
    const ExpertWeights W{W_gate_up_q, W_down_q, W_gate_up_scale, W_down_scale, Wsh_gate_up, Wsh_down};
    return forward_routed(*desc, di, x, idx, w, W, y, ws, s);
}

moe_status_t moe_backward_workspace_size(const moe_layer_desc *desc, size_t *bytes)
{
    if (!bytes)
        return MOE_ERR_INVALID_ARG;
    const moe_status_t st = check_bwd_desc(desc);
    if (st != MOE_OK)
        return st;
    *bytes = bwd_layout(*desc).total;
    return MOE_OK;
}

moe_status_t moe_backward(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wr,
                          const uint16_t *W_gate_up, const uint16_t *W_down, const uint16_t *Wsh_gate_up,
                          const uint16_t *Wsh_down, const int32_t *topk_idx, const float *topk_w, const float *dy,
                          float *dx, float *dWr, float *dW_gate_up, float *dW_down, float *dWsh_gate_up,
                          float *dWsh_down, void *ws, size_t ws_bytes, void *stream)
{
    moe_status_t st = check_bwd_desc(desc);
    if (st != MOE_OK)
        return st;
    if (desc->T == 0)
        return MOE_OK;  // nothing to do (the weight gradients of an empty batch are not written)
    const void *ptrs[] = {x, Wr, W_gate_up, W_down, Wsh_gate_up, Wsh_down, topk_idx, topk_w, dy, dx, dWr,
                          dW_gate_up, dW_down, dWsh_gate_up, dWsh_down, ws};
    for (const void *p : ptrs)
        if (!p)
            return MOE_ERR_INVALID_ARG;
    for (const void *p : ptrs)
        if (!aligned16(p))
            return MOE_ERR_UNSUPPORTED;
    const moe_layer_desc &d = *desc;
    const BwdLayout L = bwd_layout(d);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK)
        return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t *counts = at<int32_t>(ws, L.counts), *offsets = at<int32_t>(ws, L.offsets);
    int32_t *perm_token = at<int32_t>(ws, L.perm_token), *slot_of = at<int32_t>(ws, L.slot_of);
    int32_t *poff = at<int32_t>(ws, L.poff), *hdr = at<int32_t>(ws, L.hdr);
    int4 *chunks = at<int4>(ws, L.chunks), *wgroups = at<int4>(ws, L.wgroups);
    uint16_t *x_pad = at<uint16_t>(ws, L.x_pad), *dy_pad = at<uint16_t>(ws, L.dy_pad);
    float *w_pad = at<float>(ws, L.w_pad), *dw_pad = at<float>(ws, L.dw_pad), *dl_pad = at<float>(ws, L.dl_pad);
    int32_t *tok_pad = at<int32_t>(ws, L.tok_pad);
    float *gu_r = at<float>(ws, L.gu_r), *gu_s = at<float>(ws, L.gu_s);
    uint16_t *dgu_r = at<uint16_t>(ws, L.dgu_r), *dgu_s = at<uint16_t>(ws, L.dgu_s);
    uint16_t *hw_r = at<uint16_t>(ws, L.hw_r), *hw_s = at<uint16_t>(ws, L.hw_s);
    const int64_t E = d.E, H = d.H, I = d.I, Is = d.Is, P = L.P_max, Pr = L.P_r_max, Ps = L.P_s;

    // tensor maps (rows of the padded buffers are upper bounds; tiles only touch filled rows)
    CUtensorMap gu_b2, dh_b2, dx_b2_r, dx_b2_s;  // the same token rows with 128-row boxes
    CUtensorMap gu_a_r, gu_a_s, gu_b, dh_a_r, dh_a_s, dh_b, dx_a_r, dx_a_s, dx_b_r, dx_b_s, wd_a, wd_b_r, wd_b_s,
        wg_a_r, wg_a_s, wg_b, wd_o_r, wd_o_s, wg_o_r, wg_o_s;
    const bool ok = map_gate_up(&gu_a_r, W_gate_up, H, I, E, 64) && map_gate_up(&gu_a_s, Wsh_gate_up, H, Is, 1, 64) &&
                    map_rows(&gu_b, x_pad, H, P, moe::kBwdCap) && map_rows(&dh_a_r, W_down, I, E * H, 64) &&
                    map_rows(&dh_a_s, Wsh_down, Is, H, 64) && map_rows(&dh_b, dy_pad, H, P, moe::kBwdCap) &&
                    map_rows(&dx_a_r, W_gate_up, H, E * 2 * I, 64) && map_rows(&dx_a_s, Wsh_gate_up, H, 2 * Is, 64) &&
                    map_rows(&dx_b_r, dgu_r, 2 * I, Pr, moe::kBwdCap) &&
                    map_rows(&dx_b_s, dgu_s, 2 * Is, Ps, moe::kBwdCap) && map_rows(&wd_a, dy_pad, H, P, 64) &&
                    map_rows(&wd_b_r, hw_r, I, Pr, 64) && map_rows(&wd_b_s, hw_s, Is, Ps, 64) &&
                    map_rows(&wg_a_r, dgu_r, 2 * I, Pr, 64) && map_rows(&wg_a_s, dgu_s, 2 * Is, Ps, 64) &&
                    map_rows(&wg_b, x_pad, H, P, 64) && map_rows_f32_store(&wd_o_r, dW_down, I, E * H) &&
                    map_rows_f32_store(&wd_o_s, dWsh_down, Is, H) &&
                    map_rows_f32_store(&wg_o_r, dW_gate_up, H, E * 2 * I) &&
                    map_rows_f32_store(&wg_o_s, dWsh_gate_up, H, 2 * Is) &&
                    map_rows(&gu_b2, x_pad, H, P, 128) && map_rows(&dh_b2, dy_pad, H, P, 128) &&
                    map_rows(&dx_b2_r, dgu_r, 2 * I, Pr, 128) && map_rows(&dx_b2_s, dgu_s, 2 * Is, Ps, 128);
    if (!ok)
        return MOE_ERR_CUDA;
    const moe::WaitCfg wc = wait_cfg(di);
    moe::BwdArgs ba{d.T, d.H, d.E, d.k, d.I, d.Is, d.limit_routed, d.limit_shared, static_cast<int>(Ps), chunks,
                    wgroups, hdr, w_pad, tok_pad, gu_r, gu_s, dgu_r, dgu_s, hw_r, hw_s, dw_pad, dx, dW_down,
                    dW_gate_up, dWsh_down, dWsh_gate_up, counts};
    const moe::PermuteArgs pa{topk_idx, d.T, d.k, d.E, counts, offsets, perm_token, slot_of, nullptr, nullptr,
                              nullptr, nullptr, 0, di.err, 0};
    cudaError_t e = moe::launch_permute(pa, s);
    if (e == cudaSuccess)
        e = moe::launch_bwd_layout(counts, d.E, d.T, poff, chunks, wgroups, hdr, s);
    if (e == cudaSuccess)
        e = moe::launch_bwd_gather(x, dy, topk_idx, topk_w, slot_of, offsets, counts, poff, d.T, d.k, d.E, d.H,
                                   x_pad, dy_pad, w_pad, tok_pad, s);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(dw_pad, 0, static_cast<size_t>(P) * 4, s);
    if (e == cudaSuccess)
        e = moe::launch_bwd_gemm(moe::kBwdGU, gu_a_r, gu_a_s, gu_b, gu_b, gu_b2, gu_b2, ba, wc, di.num_sms, s);
    if (e == cudaSuccess)
        e = moe::launch_bwd_gemm(moe::kBwdDH, dh_a_r, dh_a_s, dh_b, dh_b, dh_b2, dh_b2, ba, wc, di.num_sms, s);
    if (e == cudaSuccess)
        e = moe::launch_bwd_router(x, Wr, topk_idx, slot_of, offsets, poff, dw_pad, d.T, d.k, d.E, d.H, d.scale,
                                   d.norm_expert_weight, dx, dl_pad, s);
    if (e == cudaSuccess)
        e = moe::launch_bwd_gemm(moe::kBwdDX, dx_a_r, dx_a_s, dx_b_r, dx_b_s, dx_b2_r, dx_b2_s, ba, wc, di.num_sms, s);
    if (e == cudaSuccess)
        e = moe::launch_bwd_gemm(moe::kBwdWD, wd_a, wd_a, wd_b_r, wd_b_s, wd_o_r, wd_o_s, ba, wc, di.num_sms, s);
    if (e == cudaSuccess)
        e = moe::launch_bwd_gemm(moe::kBwdWGU, wg_a_r, wg_a_s, wg_b, wg_b, wg_o_r, wg_o_s, ba, wc, di.num_sms, s);
    if (e == cudaSuccess)
        e = moe::launch_bwd_dwr(x_pad, dl_pad, poff, counts, d.E, d.H, dWr, s);
    return cuda_status(e);
}

moe_status_t moe_check_device(void)
{
    DeviceInfo di;
    moe_status_t st = device_info(di);
    if (st != MOE_OK)
        return st;
    if (cudaDeviceSynchronize() != cudaSuccess)
        return MOE_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpyFromSymbol(&v, g_moe_err, sizeof v) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (v != 0) {
        const uint32_t zero = 0;
        if (cudaMemcpyToSymbol(g_moe_err, &zero, sizeof zero) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    if (v & moe::kDevErrTimeout)
        return MOE_ERR_TIMEOUT;
    return (v & moe::kDevErrBounds) ? MOE_ERR_DEVICE_BOUNDS : MOE_OK;
}

moe_status_t moe_set_stage_events(void *const *events, int n)
{
    if (n < 0 || n > kMaxStageEvents || (n > 0 && !events))
        return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (!events[i])
            return MOE_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_ev_mu);
    for (int i = 0; i < n; ++i)
        g_stage_ev[i] = static_cast<cudaEvent_t>(events[i]);
    g_stage_n = n;
    return MOE_OK;
}

uint64_t moe_set_wait_limit_ns(uint64_t ns)
{
    if (ns < 1000)
        ns = 1000;
    return g_wait_limit_ns.exchange(ns);
}

}  // extern "C"
