// topk.cu -- stage 2 of the DSA decode/verify step: deterministic causal top-k.
//
// NaiveAI research page (naive.ai/en/research), "Technical Details > Hybrid
// SWA-DSA Architecture": DSA keeps the top 2,048 tokens for backbone attention.
// "NaiveRT > Why single-stream speed matters for RL": same input, bitwise-same
// output.  The selection is therefore defined as a unique set: the topk largest
// scores among s in [0, pos[t]], equal scores going to the lower position, listed
// in ascending position, -1 padded (everything when pos[t] + 1 <= topk).
//
// Method (integer arithmetic only, so it is order-independent and reproducible):
//   scores become order-preserving 32-bit keys (-0 folded onto +0);
//   hist kernel  : a 4096-bin histogram of the top 12 key bits per query
//                  (shared-memory counts, then integer global atomics);
//   select kernel: every block finds the threshold bin b1 (the bin holding the
//                  topk-th largest key) and copies the keys in bins >= b1 of its
//                  chunk, in position order, to the chunk's own region; the last
//                  block of a query (integer ticket) resolves the exact topk-th
//                  key tau with two 10-bit radix passes over those candidates,
//                  then emits, in position order, every key > tau and the first
//                  r keys == tau, r = topk - #(key > tau).
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kItems = 4;                // consecutive scores per thread per sweep
constexpr int kSmemCand = 8192;          // candidates resolved from shared memory (else from global)
constexpr int kSelectSmem = kSmemCand * 8;

// Exclusive prefix sum over the block (thread order); `total` gets the block sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t& total, uint32_t* scratch)
{
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
        uint32_t w = lane < kWarps ? scratch[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kWarps) scratch[lane] = w;
    }
    __syncthreads();
    const uint32_t before = warp ? scratch[warp - 1] : 0u;
    total = scratch[kWarps - 1];
    __syncthreads();
    return before + x - v;
}

// Find the bin b of an NB-bin histogram (bin order = key order) that holds the
// need-th largest entry: #(bins > b) < need <= #(bins >= b).  Writes b and
// #(bins > b) to res[0..1]; res[2] = 1 if found.  h may be global or shared.
template <int NB>
__device__ void find_from_top(const uint32_t* h, uint32_t need, uint32_t* res, uint32_t* scratch, bool global_h)
{
    constexpr int PER = NB / kThreads;
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
    uint32_t run = block_excl_scan(sum, total, scratch);
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

__global__ void __launch_bounds__(kThreads) topk_hist_kernel(const TopkParams p)
{
    __shared__ uint32_t h[kHistBins];
    const int t = blockIdx.y;
    const int64_t n = (int64_t)p.pos[t] + 1;
    if (n <= p.topk) return;
    const int64_t b = (int64_t)blockIdx.x * p.chunk;
    if (b >= n) return;
    const int64_t e = min(b + (int64_t)p.chunk, n);
    for (int i = threadIdx.x; i < kHistBins; i += kThreads) h[i] = 0;
    __syncthreads();
    const float* row = p.scores + (int64_t)t * p.ld;
    for (int64_t i = b + (int64_t)threadIdx.x * kItems; i < e; i += (int64_t)kThreads * kItems) {
        if (i + kItems <= e) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(row + i));
            atomicAdd(&h[score_key(v.x) >> 20], 1u);
            atomicAdd(&h[score_key(v.y) >> 20], 1u);
            atomicAdd(&h[score_key(v.z) >> 20], 1u);
            atomicAdd(&h[score_key(v.w) >> 20], 1u);
        } else {
            for (int64_t j = i; j < e; ++j) atomicAdd(&h[score_key(__ldcg(row + j)) >> 20], 1u);
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
    __shared__ uint32_t scratch[kWarps];
    __shared__ uint32_t res[3];
    __shared__ uint32_t h2[1024];
    __shared__ uint32_t off[kMaxChunks + 1];
    __shared__ uint32_t is_last;

    const int t = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x;
    const int64_t n = (int64_t)p.pos[t] + 1;
    const uint32_t topk = static_cast<uint32_t>(p.topk);
    int32_t* sel = p.sel + (int64_t)t * p.sel_ld;
    if (n <= p.topk) {   // everything visible is selected
        if (chunk == 0)
            for (int i = tid; i < p.topk; i += kThreads) sel[i] = i < n ? i : -1;
        return;
    }

    // 1. Threshold bin of the 12-bit histogram.
    find_from_top<kHistBins>(p.hist + (int64_t)t * kHistBins, topk, res, scratch, true);
    if (!res[2]) {   // histogram and scores disagree: cannot happen for consistent input
        if (tid == 0) atomicOr(p.err, ERR_TOPK_STATE);
        res[0] = 0;
        res[1] = 0;
    }
    const uint32_t b1 = res[0], gt1 = res[1];
    __syncthreads();

    // 2. Copy this chunk's keys in bins >= b1, in position order, to the chunk's region.
    const float* row = p.scores + (int64_t)t * p.ld;
    uint2* region = p.cand + (int64_t)t * p.ld + (int64_t)chunk * p.chunk;
    const int64_t b = (int64_t)chunk * p.chunk;
    const int64_t e = min(b + (int64_t)p.chunk, n);
    uint32_t run = 0;
    for (int64_t base = b; base < e; base += (int64_t)kThreads * kItems) {
        const int64_t i = base + (int64_t)tid * kItems;
        uint32_t key[kItems];
        uint32_t flags = 0, cnt = 0;
        if (i + kItems <= e) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(row + i));
            key[0] = score_key(v.x);
            key[1] = score_key(v.y);
            key[2] = score_key(v.z);
            key[3] = score_key(v.w);
#pragma unroll
            for (int j = 0; j < kItems; ++j)
                if ((key[j] >> 20) >= b1) flags |= 1u << j;
        } else {
#pragma unroll
            for (int j = 0; j < kItems; ++j) {
                key[j] = 0;
                if (i + j < e) {
                    key[j] = score_key(__ldcg(row + i + j));
                    if ((key[j] >> 20) >= b1) flags |= 1u << j;
                }
            }
        }
        cnt = __popc(flags);
        uint32_t total;
        uint32_t o = run + block_excl_scan(cnt, total, scratch);
#pragma unroll
        for (int j = 0; j < kItems; ++j)
            if (flags & (1u << j)) region[o++] = make_uint2(key[j], static_cast<uint32_t>(i + j));
        run += total;
    }
    if (tid == 0) p.counts[t * kMaxChunks + chunk] = run;

    // 3. The last block of this query finalises it.
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(p.tickets + t, 1u) == static_cast<uint32_t>(p.nchunks - 1));
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    {
        const uint32_t v = tid < p.nchunks ? __ldcg(p.counts + t * kMaxChunks + tid) : 0u;
        uint32_t m;
        const uint32_t ex = block_excl_scan(v, m, scratch);
        if (tid < p.nchunks) off[tid] = ex;
        if (tid == 0) off[p.nchunks] = m;
        __syncthreads();
    }
    const uint32_t m = off[p.nchunks];
    const uint2* cand_g = p.cand + (int64_t)t * p.ld;
    auto fetch = [&](uint32_t i) -> uint2 {
        int lo = 0, hi = p.nchunks;   // last chunk c with off[c] <= i
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (off[mid] <= i) lo = mid; else hi = mid;
        }
        return __ldcg(cand_g + (int64_t)lo * p.chunk + (i - off[lo]));
    };
    const bool in_smem = m <= static_cast<uint32_t>(kSmemCand);
    if (in_smem) {
        for (uint32_t i = tid; i < m; i += kThreads) cand_s[i] = fetch(i);
        __syncthreads();
    }
    auto get = [&](uint32_t i) -> uint2 { return in_smem ? cand_s[i] : fetch(i); };

    // Two 10-bit radix passes below the 12-bit bin give tau exactly.
    uint32_t need = topk - gt1;   // >= 1
    uint32_t prefix = b1;         // key bits resolved so far
    uint32_t above = gt1;         // keys strictly above the resolved prefix
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
        for (int i = tid; i < 1024; i += kThreads) h2[i] = 0;
        __syncthreads();
        for (uint32_t i = tid; i < m; i += kThreads) {
            const uint32_t k = get(i).x;
            if ((k >> (shift + 10)) == prefix) atomicAdd(&h2[(k >> shift) & 1023u], 1u);
        }
        __syncthreads();
        find_from_top<1024>(h2, need, res, scratch, false);
        if (!res[2]) {
            if (tid == 0) atomicOr(p.err, ERR_TOPK_STATE);
            res[0] = 0;
            res[1] = 0;
        }
        prefix = (prefix << 10) | res[0];
        above += res[1];
        need -= res[1];
        __syncthreads();
    }
    const uint32_t tau = prefix;
    const uint32_t r = need;      // keys equal to tau still to take, lowest positions first

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
                c[j] = get(i + j);
                if (c[j].x > tau) gt |= 1u << j;
                if (c[j].x == tau) eq |= 1u << j;
            }
        }
        uint32_t tie_total;
        uint32_t rank = run_tie + block_excl_scan(__popc(eq), tie_total, scratch);
        uint32_t take = gt;
#pragma unroll
        for (int j = 0; j < kItems; ++j)
            if (eq & (1u << j)) {
                if (rank < r) take |= 1u << j;
                ++rank;
            }
        uint32_t sel_total;
        uint32_t o = run_sel + block_excl_scan(__popc(take), sel_total, scratch);
#pragma unroll
        for (int j = 0; j < kItems; ++j)
            if ((take & (1u << j)) && o < topk) sel[o++] = static_cast<int32_t>(c[j].y);
        run_sel += sel_total;
        run_tie += tie_total;
    }
    if (tid == 0 && run_sel != topk) atomicOr(p.err, ERR_TOPK_STATE);
    (void)above;
}

}  // namespace

cudaError_t launch_topk_hist(const TopkParams& p, cudaStream_t s)
{
    topk_hist_kernel<<<dim3(p.nchunks, p.T), kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_topk_select(const TopkParams& p, cudaStream_t s)
{
    static int configured[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelectSmem);
        if (e != cudaSuccess) return e;
        configured[dev] = 1;
    }
    topk_select_kernel<<<dim3(p.nchunks, p.T), kThreads, kSelectSmem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace dsa
