// permute.cu — integer stages of the MoE layer on sm_100a: the token -> slot
// permutation (histogram, exclusive scan, stable scatter), the gather of token rows into
// expert-contiguous order, the tile table of the grouped GEMMs, and the fixed-order
// combine of the deterministic mode.
//
// The permutation is the local form of an expert-parallel dispatch ("MAX 中 Step-3.5-Flash
// 架构解析", section "并行模式TP_TP / TP_EP / DP_EP"): slots of expert e are
// [offsets[e], offsets[e+1]), ordered by token. Group E is the always-on shared expert
// (section "MoE共享专家、sigmoid 路由与激活裁剪") holding every token in order.
#include "internal.h"

namespace moe {
namespace {

constexpr int kPermThreads = 1024;  // 32 warps per CTA; warp w owns a contiguous token range

// Tile table of the grouped GEMMs, built by all threads of one CTA from the exclusive
// scan `offs` (E + 1 entries in shared or global memory): group g in [0, E] (E = shared
// expert, T rows) of n rows becomes ceil(n / cap) chunks of equal size rounded up to 16
// rows (the last one shorter). hdr[0] = routed chunk count, hdr[1] = total.
// The debug build checks every group's rows against `rows` (capacity of the permuted rows
// of the group's kind: T*k routed, T shared) and every entry against the table capacity.
__device__ void build_chunk_table(const int32_t *offs, int E, int T, int cap, int4 *chunks, int32_t *hdr,
                                  int max_chunks, int64_t rows, uint32_t *err)
{
    __shared__ int warp_sums[32];
    for (int g0 = 0; g0 <= E; g0 += kPermThreads) {
        // E <= 512 < kPermThreads: a single pass
        const int g = g0 + static_cast<int>(threadIdx.x);
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        int n = 0, base = 0;
        if (g < E) {
            base = offs[g];
            n = offs[g + 1] - base;
            if (!dbg_ok(base >= 0 && n >= 0 && base + static_cast<int64_t>(n) <= rows, err))
                n = 0;
        } else if (g == E) {
            n = T;
        }
        const int nch = n > 0 ? (n + cap - 1) / cap : 0;
        const int csz = nch > 0 ? ((n + nch - 1) / nch + 15) / 16 * 16 : 0;
        int incl = nch;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o)
                incl += v;
        }
        if (lane == 31)
            warp_sums[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int ws = warp_sums[lane];
            int wi = ws;
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xFFFFFFFFu, wi, o);
                if (lane >= o)
                    wi += v;
            }
            warp_sums[lane] = wi - ws;
        }
        __syncthreads();
        const int start = warp_sums[warp] + incl - nch;
        for (int c = 0; c < nch; ++c) {
            const int r = c * csz;
            const int len = n - r < csz ? n - r : csz;
            if (dbg_ok(start + c < max_chunks, err))
                chunks[start + c] = make_int4(g, base + r, len, 0);
        }
        if (g == E) {
            hdr[0] = start;
            hdr[1] = start + nch;
        }
        __syncthreads();
    }
}

// One thread-block cluster of NC CTAs (one CTA for small calls). CTA c owns a contiguous
// range of tokens; its warp w owns a contiguous sub-range.
// Pass 1: per-warp per-expert counts, built 32 entries at a time with __match_any_sync
// (one leader per distinct expert adds the group size).
// Scan: per expert, exclusive prefix over the warps of the CTA; the CTA totals meet
// through distributed shared memory, giving each CTA its base per expert and every CTA
// the global counts and their exclusive scan over experts.
// Pass 3: the same walk again; an entry's slot = offsets[e] + its CTA's base + its
// warp's base + the number of earlier lanes in its round with the same expert. Entries
// are visited in (token, rank) order, so slots within an expert are in token order: the
// result is unique and deterministic. Optionally also the per-slot routing weight and
// the grouped-GEMM tile table.
__global__ void __launch_bounds__(kPermThreads)
    permute_kernel(const PermuteArgs a)
{
    extern __shared__ int32_t sm[];
    const int E = a.E, T = a.T, k = a.k;
    int32_t *cnt = sm;            // [32][E]
    int32_t *ctot = cnt + 32 * E; // [E] this CTA's totals (read by peers)
    int32_t *cbase = ctot + E;    // [E] sum of lower CTAs' totals
    int32_t *offs = cbase + E;    // [E + 1] exclusive scan of the global counts
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int nc = static_cast<int>(gridDim.x);

    for (int i = threadIdx.x; i < 32 * E; i += kPermThreads)
        cnt[i] = 0;
    __syncthreads();

    const int per_cta = (T + nc - 1) / nc;
    const int c0 = static_cast<int>(rank) * per_cta < T ? static_cast<int>(rank) * per_cta : T;
    const int c1 = c0 + per_cta < T ? c0 + per_cta : T;
    const int per_warp = (c1 - c0 + 31) / 32;
    const int64_t t_begin = c0 + warp * per_warp < c1 ? c0 + warp * per_warp : c1;
    const int64_t t_end = t_begin + per_warp < c1 ? t_begin + per_warp : c1;
    const int64_t begin = t_begin * k, end = t_end * k;
    int32_t *mine = cnt + warp * E;

    for (int64_t b = begin; b < end; b += 32) {
        const int64_t n = b + lane;
        const bool valid = n < end;
        int e = E + lane;  // distinct sentinel for idle lanes
        if (valid) {
            e = a.idx[n];
            e = e < 0 ? 0 : (e > E - 1 ? E - 1 : e);
        }
        const unsigned m = __match_any_sync(0xFFFFFFFFu, e);
        if (valid && lane == 31 - __clz(m))
            mine[e] += __popc(m);
        __syncwarp();
    }
    __syncthreads();

    for (int e = threadIdx.x; e < E; e += kPermThreads) {
        int run = 0;
        for (int w = 0; w < 32; ++w) {
            const int c = cnt[w * E + e];
            cnt[w * E + e] = run;
            run += c;
        }
        ctot[e] = run;
    }
    cluster_sync_all();  // every CTA's totals are visible to its peers

    for (int e = threadIdx.x; e < E; e += kPermThreads) {
        int below = 0, all = 0;
        const uint32_t local = smem_u32(ctot + e);
        for (int c = 0; c < nc; ++c) {
            const int v = c == static_cast<int>(rank) ? ctot[e] : dsmem_ld_s32(dsmem_addr(local, c));
            if (c < static_cast<int>(rank))
                below += v;
            all += v;
        }
        cbase[e] = below;
        offs[e] = all;  // global count, scanned below
    }
    __syncthreads();

    if (warp == 0) {
        const int per = (E + 31) / 32;
        const int lo = lane * per;
        const int hi = lo + per < E ? lo + per : E;
        int s = 0;
        for (int e = lo; e < hi; ++e)
            s += offs[e];
        int incl = s;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o)
                incl += v;
        }
        int run = incl - s;
        for (int e = lo; e < hi; ++e) {
            const int c = offs[e];
            if (rank == 0) {
                a.counts[e] = c;
                a.offsets[e] = run;
            }
            offs[e] = run;
            run += c;
        }
        if (lane == 31) {
            offs[E] = incl;
            if (rank == 0) {
                a.counts[E] = T;
                a.offsets[E] = incl;
                a.offsets[E + 1] = incl + T;
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * E; i += kPermThreads) {
        const int e = i % E;
        cnt[i] += offs[e] + cbase[e];
    }
    __syncthreads();

    for (int64_t b = begin; b < end; b += 32) {
        const int64_t n = b + lane;
        const bool valid = n < end;
        int e = E + lane;
        if (valid) {
            e = a.idx[n];
            e = e < 0 ? 0 : (e > E - 1 ? E - 1 : e);
        }
        const unsigned m = __match_any_sync(0xFFFFFFFFu, e);
        if (valid) {
            const int slot = mine[e] + __popc(m & ((1u << lane) - 1u));
            a.slot_of[n] = slot;
            if (dbg_ok(slot >= 0 && slot < static_cast<int64_t>(T) * k, a.err)) {
                a.perm_token[slot] = static_cast<int32_t>(n / k);
                if (a.w_perm)
                    a.w_perm[slot] = a.topk_w[n];
            }
        }
        __syncwarp();
        if (valid && lane == 31 - __clz(m))
            mine[e] += __popc(m);
        __syncwarp();
    }
    const int64_t shared_base = static_cast<int64_t>(T) * k;
    for (int t = c0 + threadIdx.x; t < c1; t += kPermThreads)
        a.perm_token[shared_base + t] = t;
    if (rank == 0 && a.chunks)
        build_chunk_table(offs, E, T, a.cap, a.chunks, a.hdr, a.max_chunks, static_cast<int64_t>(T) * k, a.err);

    cluster_sync_all();  // no CTA leaves while a peer may still read its totals
}

// Per-token mode (large batches): one warp per token loads the token's row of x once (pieces
// of up to 512 16-byte vectors, all of a lane's loads in flight) and stores it into each of
// its k slots; lane j records the routing weight of slot j. x is read once instead of once per
// selected expert. Per-slot mode (small batches, where T warps would leave most of the GPU
// idle): one warp per (token, slot), x read k times (from L2). When y_zero is given, the
// warps also clear the token's row of it (the output the down GEMM then accumulates into; in
// per-slot mode slot j clears the j-th of k column ranges), in place of a separate memset.
// With amax_x, each slot also gets its row's largest |x| (float bits) and a zeroed amax_h (the
// FP8 tensor-core GEMMs scale each token row by it).
constexpr int kGatherVec = 16;        // 16-byte vectors per lane and piece
constexpr int kGatherPerTokenT = 2048;  // batches of at least this many tokens use per-token mode

// Largest magnitude among the eight bf16 of v, as bf16 magnitude bits in [0, 0x7fff] (the
// magnitude bits of non-NaN bf16 values order like the values).
__device__ __forceinline__ uint32_t bf16x8_absmax(const uint4 &v)
{
    const uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu),
                                __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu));
    return max(m & 0xffffu, m >> 16);
}

template <bool kPerSlot>
__global__ void __launch_bounds__(256)
    gather_kernel(const uint4 *__restrict__ x, const float *__restrict__ topk_w,
                  const int32_t *__restrict__ slot_of, int64_t T, int k, int vec_per_row,
                  uint4 *__restrict__ x_perm, float *__restrict__ w_perm, uint4 *__restrict__ y_zero,
                  int yvec_per_row, uint32_t *amax_x, uint32_t *amax_h, uint32_t *err)
{
    const int lane = threadIdx.x & 31;
    const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t nent = T * k;
    const int64_t units = kPerSlot ? nent : T;
    for (int64_t u = gw; u < units; u += nw) {
        const int64_t t = kPerSlot ? u / k : u;
        const int j0 = kPerSlot ? static_cast<int>(u - t * k) : 0;  // first slot of the unit
        const int nj = kPerSlot ? 1 : k;                              // slots of the unit
        // lane j < nj holds slot j0 + j of the token (the warp reads them by shuffle)
        int64_t my_slot = -1;
        if (lane < nj) {
            my_slot = slot_of[t * k + j0 + lane];
            if (!dbg_ok(my_slot >= 0 && my_slot < nent, err))
                my_slot = -1;
            else
                w_perm[my_slot] = topk_w[t * k + j0 + lane];
        }
        if (y_zero) {
            uint4 *yr = y_zero + t * yvec_per_row;
            const int c0 = kPerSlot ? static_cast<int>(static_cast<int64_t>(yvec_per_row) * j0 / k) : 0;
            const int c1 = kPerSlot ? static_cast<int>(static_cast<int64_t>(yvec_per_row) * (j0 + 1) / k)
                                    : yvec_per_row;
            for (int c = c0 + lane; c < c1; c += 32)
                yr[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        const uint4 *src = x + t * vec_per_row;
        uint32_t amax = 0;
        for (int p0 = 0; p0 < vec_per_row; p0 += 32 * kGatherVec) {
            uint4 v[kGatherVec];
#pragma unroll
            for (int i = 0; i < kGatherVec; ++i) {
                const int c = p0 + i * 32 + lane;
                if (c < vec_per_row) {
                    v[i] = __ldg(src + c);
                    if (amax_x)
                        amax = max(amax, bf16x8_absmax(v[i]));
                }
            }
            for (int j = 0; j < nj; ++j) {
                const int64_t slot = __shfl_sync(0xFFFFFFFFu, my_slot, j);
                if (slot < 0)
                    continue;
                uint4 *dst = x_perm + slot * vec_per_row;
#pragma unroll
                for (int i = 0; i < kGatherVec; ++i) {
                    const int c = p0 + i * 32 + lane;
                    if (c < vec_per_row)
                        dst[c] = v[i];
                }
            }
        }
        if (amax_x) {
            amax = __reduce_max_sync(0xFFFFFFFFu, amax);
            if (my_slot >= 0) {
                amax_x[my_slot] = amax << 16;
                amax_h[my_slot] = 0u;
            }
        }
    }
}

// Rows received by an expert-parallel dispatch ("MAX 中 Step-3.5-Flash 架构解析", section
// "并行模式TP_TP / TP_EP / DP_EP": DP_EP, each rank routes its own tokens and the experts are
// split across ranks) arrive source-major: source s sends, for each of this rank's Er experts
// in order, counts[s * Er + e] rows. The grouped GEMMs want expert-major order (expert e's
// rows from all sources contiguous), so received row n of source s at position p of that
// source's block, belonging to expert e, goes to slot
//     off[e] + col[s][e] + (p - pre[s][e])
// with off = exclusive prefix of the expert totals, col[s][e] = rows of e from sources
// before s, pre[s][e] = rows of source s for experts before e. Writes offsets [Er + 2]
// (offsets[Er] = offsets[Er + 1] = rows), perm_token[slot] = n and slot_of[n] = slot. Every
// block builds the prefix tables in shared memory; rows past the received total are skipped.
__global__ void __launch_bounds__(256)
    ep_regroup_kernel(const int32_t *__restrict__ counts, int R, int Er, int64_t nrows, int32_t *__restrict__ offsets,
                      int32_t *__restrict__ perm_token, int32_t *__restrict__ slot_of)
{
    extern __shared__ int32_t tab[];
    int32_t *src_base = tab;                 // [R + 1]
    int32_t *pre = src_base + (R + 1);       // [R][Er + 1]
    int32_t *col = pre + R * (Er + 1);       // [R][Er]
    int32_t *off = col + R * Er;             // [Er + 1]
    for (int s = threadIdx.x; s < R; s += blockDim.x) {
        int acc = 0;
        for (int e = 0; e < Er; ++e) {
            pre[s * (Er + 1) + e] = acc;
            acc += counts[s * Er + e];
        }
        pre[s * (Er + 1) + Er] = acc;
    }
    for (int e = threadIdx.x; e < Er; e += blockDim.x) {
        int acc = 0;
        for (int s = 0; s < R; ++s) {
            col[s * Er + e] = acc;
            acc += counts[s * Er + e];
        }
        off[e] = acc;  // expert total until the scan below
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int s = 0; s < R; ++s) {
            src_base[s] = acc;
            acc += pre[s * (Er + 1) + Er];
        }
        src_base[R] = acc;
        int acc2 = 0;
        for (int e = 0; e < Er; ++e) {
            const int t = off[e];
            off[e] = acc2;
            acc2 += t;
        }
        off[Er] = acc2;
        if (blockIdx.x == 0) {
            for (int e = 0; e <= Er; ++e)
                offsets[e] = off[e];
            offsets[Er + 1] = acc2;
        }
    }
    __syncthreads();
    const int64_t total = src_base[R] < nrows ? src_base[R] : nrows;
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; n < total;
         n += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        int lo = 0, hi = R - 1;  // last source whose block starts at or before n
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (src_base[mid] <= n)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int p = static_cast<int>(n - src_base[lo]);
        const int32_t *ps = pre + lo * (Er + 1);
        int a = 0, b = Er - 1;  // last expert whose rows start at or before p
        while (a < b) {
            const int mid = (a + b + 1) >> 1;
            if (ps[mid] <= p)
                a = mid;
            else
                b = mid - 1;
        }
        const int64_t slot = off[a] + col[lo * Er + a] + (p - ps[a]);
        if (slot < total) {
            perm_token[slot] = static_cast<int32_t>(n);
            slot_of[n] = static_cast<int32_t>(slot);
        }
    }
}

// Tile table from an offsets array in global memory (the moe_expert_ffn entry point).
__global__ void __launch_bounds__(kPermThreads)
    chunks_kernel(const int32_t *__restrict__ offsets, int E, int T, int cap, int4 *__restrict__ chunks,
                  int32_t *__restrict__ hdr, int cap_d, int4 *__restrict__ chunks_d, int32_t *__restrict__ hdr_d,
                  int max_chunks, int max_chunks_d, int64_t rows, uint32_t *err)
{
    build_chunk_table(offsets, E, T, cap, chunks, hdr, max_chunks, rows, err);
    if (chunks_d)
        build_chunk_table(offsets, E, T, cap_d, chunks_d, hdr_d, max_chunks_d, rows, err);
}

// y[t] = sum_{j<k} o_perm[slot_of[t, j]] + o_perm[T*k + t], in that order.
__global__ void __launch_bounds__(256)
    combine_kernel(const float4 *__restrict__ o_perm, const int32_t *__restrict__ slot_of, int T, int k,
                   int vec_per_row, float4 *__restrict__ y, uint32_t *err)
{
    const int t = blockIdx.x;
    const int64_t shared_row = static_cast<int64_t>(T) * k + t;
    for (int v = threadIdx.x; v < vec_per_row; v += blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            int64_t slot = slot_of[static_cast<int64_t>(t) * k + j];
            if (!dbg_ok(slot >= 0 && slot < static_cast<int64_t>(T) * k, err))
                continue;
            const float4 o = __ldg(o_perm + slot * vec_per_row + v);
            acc.x += o.x;
            acc.y += o.y;
            acc.z += o.z;
            acc.w += o.w;
        }
        const float4 o = __ldg(o_perm + shared_row * vec_per_row + v);
        acc.x += o.x;
        acc.y += o.y;
        acc.z += o.z;
        acc.w += o.w;
        y[static_cast<int64_t>(t) * vec_per_row + v] = acc;
    }
}

}  // namespace

cudaError_t launch_permute(const PermuteArgs &a, cudaStream_t stream)
{
    const int smem = (32 * a.E + 3 * a.E + 1) * 4;
    cudaError_t err = cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    // one CTA per 8192 (token, expert) entries, at most one portable cluster of 8
    const int64_t entries = static_cast<int64_t>(a.T) * a.k;
    int nc = static_cast<int>((entries + 8191) / 8192);
    nc = nc < 1 ? 1 : (nc > 8 ? 8 : nc);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nc, 1, 1);
    cfg.blockDim = dim3(kPermThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nc;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, permute_kernel, a);
    if (err != cudaSuccess)
        return err;
    return cudaGetLastError();
}

cudaError_t launch_gather(const uint16_t *x, const float *topk_w, const int32_t *slot_of, int T, int k, int H,
                          uint16_t *x_perm, float *w_perm, int num_sms, uint32_t *err, cudaStream_t stream,
                          float *y_zero, uint32_t *amax_x, uint32_t *amax_h)
{
    // one warp per token (or per slot), 8 warps per block, at most 8 blocks per SM
    const bool per_slot = T < kGatherPerTokenT;
    const int64_t units = per_slot ? static_cast<int64_t>(T) * k : T;
    const int64_t blocks_needed = (units + 7) / 8;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
    auto kernel = per_slot ? gather_kernel<true> : gather_kernel<false>;
    kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4 *>(x), topk_w, slot_of, T, k, H / 8,
                                     reinterpret_cast<uint4 *>(x_perm), w_perm, reinterpret_cast<uint4 *>(y_zero),
                                     H / 4, amax_x, amax_h, err);
    return cudaGetLastError();
}

size_t ep_regroup_smem(int R, int Er)
{
    return static_cast<size_t>((R + 1) + R * (Er + 1) + R * Er + (Er + 1)) * 4;
}

cudaError_t launch_ep_regroup(const int32_t *counts, int R, int Er, int64_t nrows, int32_t *offsets,
                              int32_t *perm_token, int32_t *slot_of, int num_sms, cudaStream_t stream)
{
    const size_t smem = ep_regroup_smem(R, Er);
    if (smem > 48 * 1024) {
        const cudaError_t err =
            cudaFuncSetAttribute(ep_regroup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (err != cudaSuccess)
            return err;
    }
    const int64_t need = (nrows + 255) / 256;
    const int64_t cap = static_cast<int64_t>(num_sms) * 2;
    const int grid = static_cast<int>(need < 1 ? 1 : (need < cap ? need : cap));
    ep_regroup_kernel<<<grid, 256, smem, stream>>>(counts, R, Er, nrows, offsets, perm_token, slot_of);
    return cudaGetLastError();
}

cudaError_t launch_chunks(const int32_t *offsets, int E, int T, int cap, int4 *chunks, int32_t *hdr, int cap_d,
                          int4 *chunks_d, int32_t *hdr_d, int max_chunks, int max_chunks_d, int64_t rows,
                          uint32_t *err, cudaStream_t stream)
{
    chunks_kernel<<<1, kPermThreads, 0, stream>>>(offsets, E, T, cap, chunks, hdr, cap_d, chunks_d, hdr_d, max_chunks,
                                                  max_chunks_d, rows, err);
    return cudaGetLastError();
}

cudaError_t launch_combine(const float *o_perm, const int32_t *slot_of, int T, int k, int H, float *y,
                           uint32_t *err, cudaStream_t stream)
{
    combine_kernel<<<T, 256, 0, stream>>>(reinterpret_cast<const float4 *>(o_perm), slot_of, T, k, H / 4,
                                          reinterpret_cast<float4 *>(y), err);
    return cudaGetLastError();
}

}  // namespace moe
