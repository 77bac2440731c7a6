// topk.cu -- stage 2 of the DSA decode/verify step: deterministic causal top-k.
//
// NaiveAI research page (naive.ai/en/research), "Technical Details > Hybrid
// SWA-DSA Architecture": DSA keeps the top 2,048 tokens for backbone attention.
// "NaiveRT > Why single-stream speed matters for RL": same input, bitwise-same
// output.  The selection is therefore defined as a unique set: the topk largest
// scores among s in [0, pos[t]], equal scores going to the lower position, listed
// in ascending position, -1 padded (everything when pos[t] + 1 <= topk).
//
// Method (integer arithmetic only, so it is order-independent and reproducible).
// Scores become order-preserving 32-bit keys (-0 folded onto +0).  A radix
// select over the key range [lo, hi] of the query finds the topk-th key tau:
// each pass histograms (key - lo) >> shift into 4096 bins (shift chosen so the
// range fits), keeps the bin holding the need-th largest key and narrows
// [lo, hi] to it, until one key value is left (three passes at most).  Because
// the bins follow the data's own range, keys spread over many bins and the
// shared-memory atomics rarely collide.  Emission lists every key > tau and the
// first r keys == tau (r = topk - #(key > tau)) in position order.
//
//   small n    : a cluster of 16 (or 8) blocks per query holds the keys in
//                shared memory and reduces its histograms through distributed
//                shared memory.
//   larger n   : the indexer (or a min/max kernel) leaves per-block key ranges;
//                a histogram kernel bins the first pass in global memory; a
//                select kernel copies each chunk's keys at or above the
//                threshold bin to the chunk's own region, and the last block of
//                the query (integer ticket) finishes the select on those
//                candidates and emits them in position order.
#include <cooperative_groups.h>

#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 512;            // multi-block path
constexpr int kItems = 4;                // consecutive scores per thread per sweep
constexpr int kSmemCand = 8192;          // candidates resolved from shared memory (else from global)
constexpr int kSelectSmem = kSmemCand * 8;
constexpr int kSmallThreads = 1024;      // single-block path

// Exclusive prefix sum over a block of NT threads (thread order); `total` gets
// the block sum.  scratch holds NT / 32 words.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t& total, uint32_t* scratch)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < NW ? scratch[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < NW) scratch[lane] = w;
    }
    __syncthreads();
    const uint32_t before = warp ? scratch[warp - 1] : 0u;
    total = scratch[NW - 1];
    __syncthreads();
    return before + x - v;
}

// Block-wide min of lo and max of hi (scratch holds 64 words).
template <int NT>
__device__ __forceinline__ void block_minmax(uint32_t& lo, uint32_t& hi, uint32_t* scratch)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
        scratch[warp] = lo;
        scratch[32 + warp] = hi;
    }
    __syncthreads();
    lo = scratch[0];
    hi = scratch[32];
    for (int w = 1; w < NW; ++w) {
        lo = min(lo, scratch[w]);
        hi = max(hi, scratch[32 + w]);
    }
    __syncthreads();
}

// Right shift that maps the key range [lo, hi] onto at most 4096 bins.
__device__ __forceinline__ int range_shift(uint32_t lo, uint32_t hi)
{
    const int bits = 32 - __clz(hi - lo);
    return bits > 12 ? bits - 12 : 0;
}

// Find the bin b of an NB-bin histogram (bin order = key order) that holds the
// need-th largest entry: #(bins > b) < need <= #(bins >= b).  Writes b and
// #(bins > b) to res[0..1]; res[2] = 1 if found.  h may be global or shared.
template <int NB, int NT>
__device__ void find_from_top(const uint32_t* h, uint32_t need, uint32_t* res, uint32_t* scratch, bool global_h)
{
    constexpr int PER = NB / NT;
    static_assert(PER >= 1 && NB % NT == 0, "bins must cover the block");
    const int hi = NB - PER * threadIdx.x;   // thread 0 owns the top bins
    uint32_t cnt[PER];
    uint32_t sum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        cnt[i] = global_h ? __ldcg(h + hi - 1 - i) : h[hi - 1 - i];
        sum += cnt[i];
    }
    if (threadIdx.x == 0) res[2] = 0;
    uint32_t total;
    uint32_t run = block_excl_scan<NT>(sum, total, scratch);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        if (run < need && run + cnt[i] >= need) {
            res[0] = static_cast<uint32_t>(hi - 1 - i);
            res[1] = run;
            res[2] = 1;
        }
        run += cnt[i];
    }
    __syncthreads();
}

// Radix select over n keys (read through `get`), starting from the key range
// [lo, hi] with `need` keys still to find inside it (keys above hi are already
// counted as selected, keys below lo are out).  On return lo == hi == tau and
// need = r, the number of keys equal to tau to take.
template <int NT, typename Get>
__device__ void resolve_tau(Get get, uint32_t n, uint32_t& lo, uint32_t& hi, uint32_t& need, uint32_t* hist,
                            uint32_t* res, uint32_t* scratch, uint32_t* err)
{
#pragma unroll 1
    for (int pass = 0; pass < 4 && lo != hi; ++pass) {
        const int shift = range_shift(lo, hi);
        for (int i = threadIdx.x; i < kHistBins; i += NT) hist[i] = 0;
        __syncthreads();
        for (uint32_t i = threadIdx.x; i < n; i += NT) {
            const uint32_t k = get(i);
            if (k >= lo && k <= hi) atomicAdd(&hist[(k - lo) >> shift], 1u);
        }
        __syncthreads();
        find_from_top<kHistBins, NT>(hist, need, res, scratch, false);
        if (!res[2]) {
            if (threadIdx.x == 0) atomicOr(err, ERR_TOPK_STATE);
            res[0] = 0;
            res[1] = 0;
        }
        const uint32_t b = res[0];
        need -= res[1];
        const uint32_t nlo = lo + (b << shift);
        const uint32_t width = (1u << shift) - 1u;            // shift <= 20
        hi = (nlo > 0xFFFFFFFFu - width) ? hi : min(hi, nlo + width);
        lo = nlo;
        __syncthreads();
    }
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

// A cluster of KC blocks per query; block r holds keys [r*S, (r+1)*S) of the query
// in shared memory.  Every radix pass builds block-local histograms, reduces
// them across the cluster through distributed shared memory (block r sums bin
// slice r over all blocks), and every block then finds the same threshold bin
// from the reduced slices.  The ordered emission needs only each block's
// (greater, equal) counts, exchanged the same way.
constexpr int kClusterThreads = 512;
constexpr int kClusterKeys = 12288;   // keys per block

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v);

template <int KC>
__global__ void __launch_bounds__(kClusterThreads, 1) topk_cluster_kernel(const TopkParams p)
{
    namespace cg = cooperative_groups;
    constexpr int NT = kClusterThreads;
    constexpr int SLICE = kHistBins / KC;        // bins each block reduces
    extern __shared__ __align__(16) uint32_t keys[];
    __shared__ uint32_t hist[kHistBins];
    __shared__ uint32_t slice[SLICE];           // cluster-wide sums of this block's bin slice
    __shared__ uint32_t slice_total;
    __shared__ uint32_t xchg[4];                 // lo, hi, or gt, eq published to the cluster
    __shared__ uint32_t scratch[64];
    __shared__ uint32_t res[3];
    __shared__ uint32_t w_gt[32], w_eq[32], w_sel[32], w_tie[32];
    __shared__ __align__(8) uint64_t bar;
    cg::cluster_group cluster = cg::this_cluster();

    const int rank = blockIdx.x, t = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int pos_t = 0;
#pragma unroll
    for (int i = 0; i < kMaxT; ++i)
        if (i == t) pos_t = p.pos[i];
    const int n = pos_t + 1;
    const uint32_t topk = static_cast<uint32_t>(p.topk);
    int32_t* sel = p.sel + (int64_t)t * p.sel_ld;
    // This block's positions [s0, s1); S is a multiple of 4 so rows stay 16-byte aligned.
    const int S = ((n + KC - 1) / KC + 3) & ~3;
    const int s0 = min(n, rank * S), s1 = min(n, s0 + S);
    const int cnt = s1 - s0;
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    griddep_wait();
    griddep_launch_dependents();
    if (n <= p.topk) {   // uniform over the cluster: no cluster barrier is used
        for (int i = rank * NT + tid; i < p.topk; i += KC * NT) sel[i] = i < n ? i : -1;
        return;
    }

    const int c4 = (cnt + 3) & ~3;
    if (tid == 0 && c4 > 0) {
        mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(c4) * 4u);
        bulk_g2s(keys, p.scores + (int64_t)t * p.ld + s0, static_cast<uint32_t>(c4) * 4u, &bar);
    }
    bool ok = c4 == 0 || mbar_wait(&bar, 0, p.err);
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    if (ok) {
        for (int i = tid; i < cnt; i += NT) {
            const uint32_t k = score_key(__uint_as_float(keys[i]));
            keys[i] = k;
            lo = min(lo, k);
            hi = max(hi, k);
        }
    }
    block_minmax<NT>(lo, hi, scratch);
    if (tid == 0) {
        xchg[0] = lo;
        xchg[1] = hi;
    }
    cluster.sync();
    lo = 0xFFFFFFFFu;
    hi = 0u;
#pragma unroll
    for (int r = 0; r < KC; ++r) {
        const uint32_t* x = cluster.map_shared_rank(xchg, r);
        lo = min(lo, x[0]);
        hi = max(hi, x[1]);
    }

    uint32_t need = topk;
#pragma unroll 1
    for (int pass = 0; pass < 4 && lo != hi; ++pass) {
        const int shift = range_shift(lo, hi);
        for (int i = tid; i < kHistBins; i += NT) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < cnt; i += NT) {
            const uint32_t k = keys[i];
            if (k >= lo && k <= hi) atomicAdd(&hist[(k - lo) >> shift], 1u);
        }
        cluster.sync();   // every block's histogram is complete
        // Block `rank` sums bins [rank*SLICE, (rank+1)*SLICE) over the cluster.
        for (int b = tid; b < SLICE; b += NT) {
            uint32_t v = 0;
#pragma unroll
            for (int r = 0; r < KC; ++r) v += cluster.map_shared_rank(hist, r)[rank * SLICE + b];
            slice[b] = v;
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t v = 0;
            for (int b = lane; b < SLICE; b += 32) v += slice[b];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) slice_total = v;
        }
        cluster.sync();   // every slice is reduced
        // The same search in every block: the slice, then the bin, holding the need-th largest.
        if (warp == 0) {
            uint32_t tot = lane < KC ? *cluster.map_shared_rank(&slice_total, KC - 1 - lane) : 0u;
            const uint32_t incl = warp_incl_scan(tot);   // lane j counts slices KC-1 .. KC-1-j
            const uint32_t before = incl - tot;
            const bool here = lane < KC && before < need && incl >= need;
            const uint32_t hit = __ballot_sync(0xffffffffu, here);
            const int j = hit ? __ffs(hit) - 1 : 0;
            const int sr = KC - 1 - j;                    // slice holding the threshold
            uint32_t run = __shfl_sync(0xffffffffu, before, j);
            const uint32_t* sl = cluster.map_shared_rank(slice, sr);
            int found = -1;
            uint32_t found_run = 0;
            for (int b0 = SLICE - 32; b0 >= 0 && found < 0; b0 -= 32) {   // 32 bins at a time, top down
                const uint32_t v = sl[b0 + 31 - lane];
                const uint32_t vi = warp_incl_scan(v);
                const uint32_t bb = run + vi - v;
                const uint32_t h2 = __ballot_sync(0xffffffffu, bb < need && bb + v >= need);
                if (h2) {
                    const int l2 = __ffs(h2) - 1;
                    found = sr * SLICE + b0 + 31 - l2;
                    found_run = __shfl_sync(0xffffffffu, bb, l2);
                }
                run += __shfl_sync(0xffffffffu, vi, 31);
            }
            if (lane == 0) {
                if (!hit || found < 0) {
                    atomicOr(p.err, ERR_TOPK_STATE);
                    found = 0;
                    found_run = 0;
                }
                res[0] = static_cast<uint32_t>(found);
                res[1] = found_run;
            }
        }
        __syncthreads();
        const uint32_t b = res[0];
        need -= res[1];
        const uint32_t nlo = lo + (b << shift);
        const uint32_t width = (1u << shift) - 1u;
        hi = (nlo > 0xFFFFFFFFu - width) ? hi : min(hi, nlo + width);
        lo = nlo;
    }
    const uint32_t tau = lo, r = need;

    // Per-warp (greater, equal) counts of this block's contiguous warp segments.
    constexpr int NW = NT / 32;
    const int seg = ((cnt + NW - 1) / NW + 31) / 32 * 32;
    const int wlo = min(cnt, warp * seg), whi = min(cnt, wlo + seg);
    uint32_t gt = 0, eq = 0;
    for (int i = wlo + lane; i < whi; i += 32) {
        gt += keys[i] > tau;
        eq += keys[i] == tau;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gt += __shfl_xor_sync(0xffffffffu, gt, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0) {
        w_gt[warp] = gt;
        w_eq[warp] = eq;
    }
    __syncthreads();
    if (warp == 0) {
        const uint32_t g = lane < NW ? w_gt[lane] : 0u, e = lane < NW ? w_eq[lane] : 0u;
        const uint32_t gs = warp_incl_scan(g), es = warp_incl_scan(e);
        if (lane == 31) {
            xchg[2] = gs;
            xchg[3] = es;
        }
    }
    cluster.sync();   // every block's totals are published
    if (warp == 0) {
        // Ties before this block, and outputs before it, from the blocks ranked below.
        uint32_t g = 0, e = 0;
        if (lane < KC) {
            const uint32_t* x = cluster.map_shared_rank(xchg, lane);
            g = x[2];
            e = x[3];
        }
        const uint32_t e_before = warp_incl_scan(e) - e;
        const uint32_t taken = e_before >= r ? 0u : min(e, r - e_before);
        const uint32_t o_before = warp_incl_scan(g + taken) - (g + taken);
        const uint32_t tie_base = __shfl_sync(0xffffffffu, e_before, rank);
        const uint32_t out_base = __shfl_sync(0xffffffffu, o_before, rank);
        // Then per warp of this block.
        const uint32_t we = lane < NW ? w_eq[lane] : 0u;
        const uint32_t wtb = tie_base + warp_incl_scan(we) - we;
        const uint32_t wtaken = wtb >= r ? 0u : min(we, r - wtb);
        const uint32_t wg = (lane < NW ? w_gt[lane] : 0u) + wtaken;
        const uint32_t wob = out_base + warp_incl_scan(wg) - wg;
        if (lane < NW) {
            w_tie[lane] = wtb;
            w_sel[lane] = wob;
        }
    }
    __syncthreads();
    uint32_t tie_run = w_tie[warp], sel_run = w_sel[warp];
    for (int base = wlo; base < whi; base += 32) {
        const int i = base + lane;
        const uint32_t k = i < whi ? keys[i] : 0u;
        const bool g = i < whi && k > tau, e = i < whi && k == tau;
        const uint32_t lt = (1u << lane) - 1u;
        const uint32_t eb = __ballot_sync(0xffffffffu, e);
        const bool take = g || (e && tie_run + __popc(eb & lt) < r);
        const uint32_t tb = __ballot_sync(0xffffffffu, take);
        if (take) {
            const uint32_t o = sel_run + __popc(tb & lt);
            if (o < topk) sel[o] = s0 + i;
        }
        tie_run += __popc(eb);
        sel_run += __popc(tb);
    }
    if (!ok && tid == 0) mbar_wait(&bar, 0, p.err);
    cluster.sync();   // no block leaves while its shared memory may still be read
}

// Key range [lo, hi] of query t from the per-block ranges the producer left.
__device__ __forceinline__ void query_range(const TopkParams& p, int t, uint32_t& lo, uint32_t& hi, uint32_t* scratch)
{
    lo = 0xFFFFFFFFu;
    hi = 0u;
    for (int i = threadIdx.x; i < p.mm_slots; i += kThreads) {
        const uint2 v = __ldcg(reinterpret_cast<const uint2*>(p.mm) + (int64_t)i * kMaxT + t);
        lo = min(lo, v.x);
        hi = max(hi, v.y);
    }
    block_minmax<kThreads>(lo, hi, scratch);
}

// Per-block key ranges of every query (used when no indexer produced them).
__global__ void __launch_bounds__(kThreads) topk_minmax_kernel(const TopkParams p)
{
    __shared__ uint32_t scratch[64];
    const int t = blockIdx.y;
    const int64_t n = (int64_t)p.pos[t] + 1;
    griddep_wait();
    griddep_launch_dependents();
    const int64_t b = (int64_t)blockIdx.x * p.chunk;
    const int64_t e = min(b + (int64_t)p.chunk, n);
    const float* row = p.scores + (int64_t)t * p.ld;
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (int64_t i = b + threadIdx.x; i < e; i += kThreads) {
        const uint32_t k = score_key(__ldcg(row + i));
        lo = min(lo, k);
        hi = max(hi, k);
    }
    block_minmax<kThreads>(lo, hi, scratch);
    if (threadIdx.x == 0) reinterpret_cast<uint2*>(p.mm)[(int64_t)blockIdx.x * kMaxT + t] = make_uint2(lo, hi);
}

__global__ void __launch_bounds__(kThreads) topk_hist_kernel(const TopkParams p)
{
    __shared__ uint32_t h[kHistBins];
    __shared__ uint32_t scratch[64];
    const int t = blockIdx.y;
    const int64_t n = (int64_t)p.pos[t] + 1;
    griddep_wait();
    griddep_launch_dependents();
    if (n <= p.topk) return;
    const int64_t b = (int64_t)blockIdx.x * p.chunk;
    if (b >= n) return;
    const int64_t e = min(b + (int64_t)p.chunk, n);
    uint32_t lo, hi;
    query_range(p, t, lo, hi, scratch);
    const int shift = range_shift(lo, hi);
    for (int i = threadIdx.x; i < kHistBins; i += kThreads) h[i] = 0;
    __syncthreads();
    const float* row = p.scores + (int64_t)t * p.ld;
    for (int64_t i = b + (int64_t)threadIdx.x * kItems; i < e; i += (int64_t)kThreads * kItems) {
        if (i + kItems <= e) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(row + i));
            atomicAdd(&h[(score_key(v.x) - lo) >> shift], 1u);
            atomicAdd(&h[(score_key(v.y) - lo) >> shift], 1u);
            atomicAdd(&h[(score_key(v.z) - lo) >> shift], 1u);
            atomicAdd(&h[(score_key(v.w) - lo) >> shift], 1u);
        } else {
            for (int64_t j = i; j < e; ++j) atomicAdd(&h[(score_key(__ldcg(row + j)) - lo) >> shift], 1u);
        }
    }
    __syncthreads();
    uint32_t* gh = p.hist + (int64_t)t * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += kThreads)
        if (h[i]) atomicAdd(gh + i, h[i]);
}

__global__ void __launch_bounds__(kThreads) topk_select_kernel(const TopkParams p)
{
    extern __shared__ uint2 cand_s[];            // kSmemCand candidates (finalising block only)
    __shared__ uint32_t scratch[64];
    __shared__ uint32_t res[3];
    __shared__ uint32_t h2[kHistBins];
    __shared__ uint32_t off[kMaxChunks + 1];
    __shared__ uint32_t is_last;

    const int t = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x;
    const int64_t n = (int64_t)p.pos[t] + 1;
    const uint32_t topk = static_cast<uint32_t>(p.topk);
    int32_t* sel = p.sel + (int64_t)t * p.sel_ld;
    griddep_wait();
    griddep_launch_dependents();
    if (n <= p.topk) {   // everything visible is selected
        if (chunk == 0)
            for (int i = tid; i < p.topk; i += kThreads) sel[i] = i < n ? i : -1;
        return;
    }

    // 1. The first pass's threshold bin b1 from the global histogram.
    uint32_t lo, hi;
    query_range(p, t, lo, hi, scratch);
    const int shift = range_shift(lo, hi);
    find_from_top<kHistBins, kThreads>(p.hist + (int64_t)t * kHistBins, topk, res, scratch, true);
    if (!res[2]) {   // histogram and scores disagree: cannot happen for consistent input
        if (tid == 0) atomicOr(p.err, ERR_TOPK_STATE);
        res[0] = 0;
        res[1] = 0;
    }
    const uint32_t b1 = res[0], gt1 = res[1];
    const uint32_t cut = lo + (b1 << shift);   // every key >= cut is a candidate
    __syncthreads();

    // 2. Copy this chunk's keys >= cut, in position order, to the chunk's region.
    const float* row = p.scores + (int64_t)t * p.ld;
    uint2* region = p.cand + (int64_t)t * p.ld + (int64_t)chunk * p.chunk;
    const int64_t b = (int64_t)chunk * p.chunk;
    const int64_t e = min(b + (int64_t)p.chunk, n);
    uint32_t run = 0;
    for (int64_t base = b; base < e; base += (int64_t)kThreads * kItems) {
        const int64_t i = base + (int64_t)tid * kItems;
        uint32_t key[kItems];
        uint32_t flags = 0;
        if (i + kItems <= e) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(row + i));
            key[0] = score_key(v.x);
            key[1] = score_key(v.y);
            key[2] = score_key(v.z);
            key[3] = score_key(v.w);
#pragma unroll
            for (int j = 0; j < kItems; ++j)
                if (key[j] >= cut) flags |= 1u << j;
        } else {
#pragma unroll
            for (int j = 0; j < kItems; ++j) {
                key[j] = 0;
                if (i + j < e) {
                    key[j] = score_key(__ldcg(row + i + j));
                    if (key[j] >= cut) flags |= 1u << j;
                }
            }
        }
        uint32_t total;
        uint32_t o = run + block_excl_scan<kThreads>(__popc(flags), total, scratch);
#pragma unroll
        for (int j = 0; j < kItems; ++j)
            if (flags & (1u << j)) region[o++] = make_uint2(key[j], static_cast<uint32_t>(i + j));
        run += total;
    }
    if (tid == 0) p.counts[t * kMaxChunks + chunk] = run;

    // 3. The last block of this query finishes it.
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(p.tickets + t, 1u) == static_cast<uint32_t>(p.nchunks - 1));
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    {
        const uint32_t v = tid < p.nchunks ? __ldcg(p.counts + t * kMaxChunks + tid) : 0u;
        uint32_t m;
        const uint32_t ex = block_excl_scan<kThreads>(v, m, scratch);
        if (tid < p.nchunks) off[tid] = ex;
        if (tid == 0) off[p.nchunks] = m;
        __syncthreads();
    }
    const uint32_t m = off[p.nchunks];
    const uint2* cand_g = p.cand + (int64_t)t * p.ld;
    const bool in_smem = m <= static_cast<uint32_t>(kSmemCand);
    if (in_smem) {   // warp w copies chunks w, w + 16, ... (coalesced, independent)
        const int warp = tid >> 5, lane = tid & 31;
        for (int c = warp; c < p.nchunks; c += kThreads / 32) {
            const uint32_t c0 = off[c], cnt = off[c + 1] - c0;
            for (uint32_t i = lane; i < cnt; i += 32) cand_s[c0 + i] = __ldcg(cand_g + (int64_t)c * p.chunk + i);
        }
        __syncthreads();
    }
    auto fetch = [&](uint32_t i) -> uint2 {
        if (in_smem) return cand_s[i];
        int a = 0, z = p.nchunks;   // last chunk c with off[c] <= i
        while (z - a > 1) {
            const int mid = (a + z) >> 1;
            if (off[mid] <= i) a = mid; else z = mid;
        }
        return __ldcg(cand_g + (int64_t)a * p.chunk + (i - off[a]));
    };

    // Finish the select inside the threshold bin's key range.
    uint32_t rlo = cut;
    const uint32_t width = (1u << shift) - 1u;
    uint32_t rhi = (cut > 0xFFFFFFFFu - width) ? hi : min(hi, cut + width);
    uint32_t need = topk - gt1;
    resolve_tau<kThreads>([&](uint32_t i) { return fetch(i).x; }, m, rlo, rhi, need, h2, res, scratch, p.err);
    const uint32_t tau = rlo;
    const uint32_t r = need;

    // Ordered emission: candidates are already in ascending position.
    uint32_t run_sel = 0, run_tie = 0;
    for (uint32_t base = 0; base < m; base += kThreads * kItems) {
        const uint32_t i = base + tid * kItems;
        uint2 c[kItems];
        uint32_t eq = 0, gt = 0;
#pragma unroll
        for (int j = 0; j < kItems; ++j) {
            c[j] = make_uint2(0u, 0u);
            if (i + j < m) {
                c[j] = fetch(i + j);
                if (c[j].x > tau) gt |= 1u << j;
                if (c[j].x == tau) eq |= 1u << j;
            }
        }
        uint32_t tie_total;
        uint32_t rank = run_tie + block_excl_scan<kThreads>(__popc(eq), tie_total, scratch);
        uint32_t take = gt;
#pragma unroll
        for (int j = 0; j < kItems; ++j)
            if (eq & (1u << j)) {
                if (rank < r) take |= 1u << j;
                ++rank;
            }
        uint32_t sel_total;
        uint32_t o = run_sel + block_excl_scan<kThreads>(__popc(take), sel_total, scratch);
#pragma unroll
        for (int j = 0; j < kItems; ++j)
            if ((take & (1u << j)) && o < topk) sel[o++] = static_cast<int32_t>(c[j].y);
        run_sel += sel_total;
        run_tie += tie_total;
    }
    if (tid == 0 && run_sel != topk) atomicOr(p.err, ERR_TOPK_STATE);
}

int g_topk_cluster[64] = {};
bool g_select_configured[64] = {};

}  // namespace

int topk_cluster_size()
{
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 8;
    if (g_topk_cluster[dev]) return g_topk_cluster[dev];
    const int smem = kClusterKeys * 4;
    cudaFuncSetAttribute(topk_cluster_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    cudaFuncSetAttribute(topk_cluster_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncSetAttribute(topk_cluster_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16, 1, 1);
    cfg.blockDim = dim3(kClusterThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 16;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const bool ok16 = cudaOccupancyMaxActiveClusters(&n, topk_cluster_kernel<16>, &cfg) == cudaSuccess && n >= 1;
    cudaGetLastError();
    g_topk_cluster[dev] = ok16 ? 16 : 8;
    return g_topk_cluster[dev];
}

int64_t topk_cluster_capacity() { return (int64_t)topk_cluster_size() * (kClusterKeys - 4); }

cudaError_t launch_topk_cluster(const TopkParams& p, cudaStream_t s)
{
    const int KC = topk_cluster_size();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(KC, p.T, 1);
    cfg.blockDim = dim3(kClusterThreads, 1, 1);
    cfg.dynamicSmemBytes = kClusterKeys * 4;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = KC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return KC == 16 ? cudaLaunchKernelEx(&cfg, topk_cluster_kernel<16>, p)
                    : cudaLaunchKernelEx(&cfg, topk_cluster_kernel<8>, p);
}

cudaError_t launch_topk_minmax(const TopkParams& p, cudaStream_t s)
{
    return launch_pdl(topk_minmax_kernel, dim3(p.nchunks, p.T), dim3(kThreads), 0, s, p);
}

cudaError_t launch_topk_hist(const TopkParams& p, cudaStream_t s)
{
    return launch_pdl(topk_hist_kernel, dim3(p.nchunks, p.T), dim3(kThreads), 0, s, p);
}

cudaError_t launch_topk_select(const TopkParams& p, cudaStream_t s)
{
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !g_select_configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelectSmem);
        if (e != cudaSuccess) return e;
        g_select_configured[dev] = true;
    }
    return launch_pdl(topk_select_kernel, dim3(p.nchunks, p.T), dim3(kThreads), kSelectSmem, s, p);
}

}  // namespace dsa
