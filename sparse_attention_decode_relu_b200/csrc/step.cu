// step.cu -- the DSA decode/verify step as two persistent kernels.
//
// NaiveAI research page (naive.ai/en/research), "NaiveRT > A DSA layer: from 29
// kernels to one": a DSA layer runs as a single cooperative kernel across 148
// CTAs in one grid.  Here one block per SM runs the step in two launches:
//
//   1 index   : (index_kernel) ReLU indexer scan over the key cache,
//               warp-specialised on the fifth-generation tensor cores (TMA key
//               tiles, FP8 keys widened into tensor memory, tcgen05.mma, an
//               epilogue that writes fp32 scores, per-32-position key maxima and
//               a lower-bound histogram of the keys' top 12 bits -- the first
//               radix pass of the top-k)
//   -- step_kernel, a cooperative programmatic dependent of the first: its
//      blocks wait for the whole indexer grid, no grid barrier of their own --
//   2 extract : per (query, chunk): every score whose key reaches the query's
//               cut bin goes to a candidate sub-segment, in position order
//   3 select  : per query (block t): the exact top-k among the candidates, ties
//               to the lower position, written in ascending order; a release
//               flag per query
//   (or)      : selection by position: the last W visible positions (the
//               short-context bypass with W = topk, sliding-window decode)
//   4 attend  : gathered sparse attention per (query, row split), each item
//               starting as soon as its query's selection is flagged: whole
//               K/V rows by bulk async copy, tensor-core QK and PV, online
//               softmax; partial (max, sum, output) states to global memory
//   5 merge   : per (query, head), the splits merged in a fixed order, as soon
//               as every split of the query is done
//
// Stage entry points run a sub-range of the phases (caller scores: the exact
// histogram in step_kernel, then one grid barrier before the extraction).  Every reduction is either
// integer or in a fixed order, so results are bitwise reproducible.
#include <type_traits>

#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;

// ---- shared memory map (dynamic, 1024-aligned base) --------------------------
constexpr int kTileRows = 16;             // K/V rows per attention tile (the n side of an m16n8k16 MMA)
constexpr int kDataBytes = 200 * 1024;    // the phases' data region; each phase lays out its own buffers
constexpr int kBarOffset = (kDataBytes + 127) / 128 * 128;
constexpr int kBarSlots = 96;             // mbarriers (8 bytes each) after the data region
constexpr int kStepSmem = 1024 + kBarOffset + kBarSlots * 8;

// mbarrier slots of each phase (disjoint, so no phase re-initialises another's)
constexpr int kBarRawFull = 0, kBarAFull = 8, kBarAEmpty = 12, kBarAccFull = 16, kBarAccEmpty = 19, kBarRawEmpty = 22,
              kBarSetup = 30;
constexpr int kBarExtract = 32;           // [8 warps][4 stages]
constexpr int kBarAttFull = 64, kBarAttEmpty = 80;


__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Spin (one thread) until *word >= target + p.barrier_extra, bounded by
// p.barrier_limit SM clocks (error bit and false when it runs out).
__device__ bool wait_counter(const StepParams& p, const uint32_t* word, uint32_t target)
{
    target += p.barrier_extra;
    if (ld_acquire(word) >= target) return true;
    const long long t0 = clock64();
    while (ld_acquire(word) < target) {
        if (clock64() - t0 > p.barrier_limit) {
            atomicOr(p.err, ERR_WAIT_TIMEOUT);
            return false;
        }
        // Hundreds of waiters poll words of one 128-byte line: a pause between polls
        // keeps that L2 slice free for the data the others are moving.
        __nanosleep(200);
    }
    return true;
}

// Grid-wide barrier among the co-resident blocks of a cooperative launch.  The
// arrival counter only grows during a launch (it is zero at launch): barrier k
// ends when it reaches k * gridDim.x.  Each block adds 1 with release semantics
// and polls with acquire loads, giving up (error bit, false) after
// p.barrier_limit SM clocks.  The launch leaves its control words at zero again
// (see barrier_exit), so consecutive launches need no reset node.
struct GridBarrier {
    uint32_t* count;
    uint32_t next;     // count value that ends the next barrier
    uint32_t c0 = 0, x0 = 0;   // (thread 0) arrival and exit words as this block first saw them
    bool bad = false;          // (thread 0) they were not zero at launch

    // Thread 0 reads the control words at kernel entry; they are checked at the
    // first barrier, so the loads overlap the first phase.
    __device__ void enter()
    {
        if (threadIdx.x == 0) {
            c0 = *reinterpret_cast<volatile uint32_t*>(count);
            x0 = *reinterpret_cast<volatile uint32_t*>(count + kCtrlWordExit);
        }
    }

    __device__ bool sync(const StepParams& p, int* ok_s)
    {
        __syncthreads();
        if (threadIdx.x == 0) {
            // Before its first arrival a block can see at most gridDim.x - 1
            // arrivals and no exit (nobody passes the first barrier without it);
            // anything else means the words were not zero at launch.  Such a
            // block flags it and takes no part in the barriers.
            if (next == gridDim.x && (x0 != 0u || c0 >= gridDim.x)) {
                bad = true;
                atomicOr(p.err, ERR_WORKSPACE_STATE);
            }
            bool ok = !bad;
            if (ok) {
                red_release_add(count, 1u);
                ok = wait_counter(p, count, next);
            }
            *ok_s = ok ? 1 : 0;
        }
        __syncthreads();
        next += gridDim.x;
        return *ok_s != 0;
    }
};

// Every block counts itself out (a release add, no round trip); block 0 waits
// for the whole grid, then resets every control word but the epoch and advances
// the epoch (which histogram buffer the next launch uses).  A returning atomic
// on one word from every block serialises for microseconds; this costs one
// bounded wait in one block.  If that wait runs out the words stay as they are,
// and the next launch on the workspace reports them.
__device__ __forceinline__ void barrier_exit(const StepParams& p)
{
    if (threadIdx.x == 0) {
        red_release_add(p.ctrl + kCtrlWordExit, 1u);
        if (blockIdx.x == 0) {
            const uint32_t* word = p.ctrl + kCtrlWordExit;
            bool ok = ld_acquire(word) >= gridDim.x;
            const long long t0 = clock64();
            while (!ok) {
                if (clock64() - t0 > kWaitLimitCycles) {   // (not shortened by the test hook)
                    atomicOr(p.err, ERR_WAIT_TIMEOUT);
                    break;
                }
                ok = ld_acquire(word) >= gridDim.x;
            }
            if (ok) {
                p.ctrl[0] = 0u;
                p.ctrl[kCtrlWordExit] = 0u;
                p.ctrl[kCtrlWordBad] = 0u;
                for (int t = 0; t < kMaxT; ++t) {
                    p.ctrl[kCtrlWordArrive + t] = 0u;
                    p.ctrl[kCtrlWordReady + t] = 0u;
                    p.ctrl[kCtrlWordDone + t] = 0u;
                }
                p.ctrl[kCtrlWordEpoch] += 1u;
                __threadfence();
            }
        }
    }
}

// The control words are zero at launch but for the epoch (the previous launch on
// the workspace left them so).  The indexer kernel checks them for the
// cooperative kernel that follows it, before any of its blocks can write one
// (they wait for the whole indexer grid first); if they are not, it flags the
// workspace state and marks the words bad, and that kernel skips its phases.
// The mark is written either way, so a stale one does not outlive the check.
__device__ void check_ctrl_words(const StepParams& p)
{
    uint32_t any = *reinterpret_cast<volatile uint32_t*>(p.ctrl) | *reinterpret_cast<volatile uint32_t*>(p.ctrl + kCtrlWordExit);
    for (int t = 0; t < kMaxT; ++t)
        any |= *reinterpret_cast<volatile uint32_t*>(p.ctrl + kCtrlWordArrive + t) |
               *reinterpret_cast<volatile uint32_t*>(p.ctrl + kCtrlWordReady + t) |
               *reinterpret_cast<volatile uint32_t*>(p.ctrl + kCtrlWordDone + t);
    if (any != 0u) atomicOr(p.err, ERR_WORKSPACE_STATE);
    p.ctrl[kCtrlWordBad] = any != 0u ? 1u : 0u;
}

// Per-launch state every block reads at entry.
struct LaunchView {
    int32_t pos[kMaxT];      // query positions (device memory; the launch parameters otherwise)
    int32_t n_max;           // furthest visible position + 1
    uint32_t* hist;          // this launch's global histogram [kMaxT][kHistBins], or nullptr
};
__shared__ LaunchView g_view;

__device__ __forceinline__ int query_pos(const StepParams& p, int k)
{
    return p.pos_dev != nullptr ? g_view.pos[k] : p.pos[k];
}
__device__ __forceinline__ int visible_max(const StepParams& p)
{
    return p.pos_dev != nullptr ? g_view.n_max : p.n_max;
}
// Position of query t for a run-time t (unrolled selection, no local memory).
__device__ __forceinline__ int query_pos_rt(const StepParams& p, int t)
{
    int v = 0;
#pragma unroll
    for (int k = 0; k < kMaxT; ++k)
        if (k == t) v = query_pos(p, k);
    return v;
}

// Phase-boundary timestamp (when the caller asked for a trace).
__device__ __forceinline__ void stamp(const StepParams& p, int slot)
{
    if (p.trace != nullptr && threadIdx.x == 0) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        p.trace[(int64_t)blockIdx.x * kTraceSlots + slot] = t;
    }
}

// ---- block-wide helpers ----------------------------------------------------------
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

// Exclusive prefix sum over the block (thread order); `total` gets the sum.
// One barrier between the warp scans and every thread summing the eight warp
// totals itself (two 16-byte reads), one more before scratch is reused.
// scratch: 16-byte aligned.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t& total, uint32_t* scratch)
{
    static_assert(kWarps == 8, "two 16-byte reads of warp totals");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t x = warp_incl_scan(v);
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    const uint4 a = reinterpret_cast<const uint4*>(scratch)[0], b = reinterpret_cast<const uint4*>(scratch)[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        tot += w[i];
        before += i < warp ? w[i] : 0u;
    }
    total = tot;
    __syncthreads();
    return before + x - v;
}

// Exclusive prefix maximum over the block (thread order; 0 for thread 0).
__device__ __forceinline__ uint32_t block_excl_max(uint32_t v, uint32_t* scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x = max(x, y);
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    uint32_t before = 0;
    for (int w = 0; w < warp; ++w) before = max(before, scratch[w]);
    const uint32_t prev = __shfl_up_sync(0xffffffffu, x, 1);
    if (lane > 0) before = max(before, prev);
    __syncthreads();
    return before;
}

// In-place exclusive prefix sum of a[0, n) in shared memory (each thread scans
// a contiguous run); returns the total.
__device__ uint32_t block_scan_array(uint32_t* a, int n, uint32_t* scratch)
{
    const int per = (n + kThreads - 1) / kThreads;
    const int j0 = min(n, static_cast<int>(threadIdx.x) * per), j1 = min(n, j0 + per);
    uint32_t s = 0;
    for (int j = j0; j < j1; ++j) s += a[j];
    uint32_t total;
    uint32_t run = block_excl_scan(s, total, scratch);
    for (int j = j0; j < j1; ++j) {
        const uint32_t v = a[j];
        a[j] = run;
        run += v;
    }
    __syncthreads();
    return total;
}

// Work item i of `items` assigned to this block in round r (i = block + r*grid).
__device__ __forceinline__ int item_of(int r) { return blockIdx.x + r * gridDim.x; }

// Right shift that maps the key range [lo, hi] onto at most 4096 bins.
__device__ __forceinline__ int range_shift(uint32_t lo, uint32_t hi)
{
    const int bits = 32 - __clz(hi - lo);
    return bits > 12 ? bits - 12 : 0;
}

// Highest key of the bin that starts at `start` (bins of width 2^shift), clamped to hi.
__device__ __forceinline__ uint32_t bin_top(uint32_t start, int shift, uint32_t hi)
{
    const uint32_t width = (1u << shift) - 1u;   // shift <= 24
    return (start > 0xFFFFFFFFu - width) ? hi : min(hi, start + width);
}

// Bin b of a kHistBins-bin histogram in shared memory holding the need-th
// largest entry: #(bins > b) < need <= #(bins >= b).  res = {b, #(bins > b),
// found}.  The bins form 128 chunks of 32; every warp sums its chunks (lane l
// reads bin 32c + l: no bank conflicts); warp 0 then scans the chunk sums from
// the top, and the chosen chunk's bins from the top.
__device__ void find_from_top(const uint32_t* h, uint32_t need, uint32_t* res)
{
    constexpr int kChunks = kHistBins / 32;
    __shared__ uint32_t csum[kChunks];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int c = warp; c < kChunks; c += kWarps) {
        const uint32_t v = __reduce_add_sync(0xffffffffu, h[c * 32 + lane]);
        if (lane == 0) csum[c] = v;
    }
    __syncthreads();
    if (warp == 0) {
        // lane l takes chunks 127 - 4l .. 124 - 4l, i.e. from the top
        uint32_t cs[4], sum = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            cs[j] = csum[kChunks - 1 - 4 * lane - j];
            sum += cs[j];
        }
        const uint32_t incl = warp_incl_scan(sum);
        uint32_t run = incl - sum;
        int chunk = -1;
        uint32_t before = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (run < need && run + cs[j] >= need) {
                chunk = kChunks - 1 - 4 * lane - j;
                before = run;
            }
            run += cs[j];
        }
        const uint32_t who = __ballot_sync(0xffffffffu, chunk >= 0);
        if (who) {
            const int src = __ffs(who) - 1;
            chunk = __shfl_sync(0xffffffffu, chunk, src);
            before = __shfl_sync(0xffffffffu, before, src);
            const int bin = chunk * 32 + 31 - lane;   // lane l: the chunk's bins from the top
            const uint32_t v = h[bin];
            const uint32_t vi = warp_incl_scan(v);
            const uint32_t ex = before + vi - v;
            if (ex < need && ex + v >= need) {
                res[0] = static_cast<uint32_t>(bin);
                res[1] = ex;
                res[2] = 1;
            }
        } else if (lane == 0) {
            res[2] = 0;
        }
    }
    __syncthreads();
}

// One radix pass over keys in [lo, hi]: count(f) adds each key of the pass's
// input to the shared histogram h through the callback; the bin holding the
// need-th largest key becomes the new [lo, hi] and need is reduced by the keys
// above it.  When lo == hi the key is exact and need = how many entries equal
// to it are to be taken.
template <typename ForEach>
__device__ void radix_pass(ForEach for_each_key, uint32_t& lo, uint32_t& hi, uint32_t& need, uint32_t* h,
                           uint32_t* res, uint32_t* scratch, uint32_t* err)
{
    const int shift = range_shift(lo, hi);
    for (int b = threadIdx.x; b < kHistBins; b += kThreads) h[b] = 0u;
    __syncthreads();
    const uint32_t l0 = lo, h0 = hi;
    for_each_key([&](uint32_t k) {
        if (k >= l0 && k <= h0) atomicAdd(&h[(k - l0) >> shift], 1u);
    });
    __syncthreads();
    find_from_top(h, need, res);
    if (!res[2]) {
        if (threadIdx.x == 0) atomicOr(err, ERR_TOPK_STATE);
        res[0] = 0;
        res[1] = 0;
    }
    const uint32_t nlo = lo + (res[0] << shift);
    hi = bin_top(nlo, shift, hi);
    lo = nlo;
    need -= res[1];
    __syncthreads();
}

// ==================================================================================
// Phase 1: indexer scan on the fifth-generation tensor cores, a kernel of its own
// with 17 warps per SM in three roles, decoupled by tensor-memory buffers so that
// each runs at its own pace.  A tile of 128 keys is the M side of tcgen05.mma
// kind::f16 (bf16 operands, fp32 accumulators in tensor memory), the T x 16
// indexer query heads the N side (16..128), the 64 dims K (four K = 16 steps).
//   - Warps 0-3, one per TMEM lane quarter (32 key rows): (FP8 keys) widen each
//     row's 64 E4M3 codes (TMA tile, 64-byte swizzle) exactly into f16 (one
//     conversion instruction per two codes), straight into the tile's
//     tensor-memory A buffer (four of them); bf16 keys arrive from TMA already as
//     the shared-memory A operand (128-byte swizzle).
//   - Warp 16: one thread issues tile j's MMAs once its A operand is in and its
//     accumulator buffer is free, and refills the TMA ring.
//   - Warps 4-15, three per lane quarter: the epilogue of queries [e T / 3, (e +
//     1) T / 3) for the e-th of them: load the accumulator columns, release the
//     buffer, then ReLU, head weights, a fixed-order sum over the 16 heads, the
//     per-token scale; the fp32 score goes to global memory, the largest key of
//     each 32-position group (per query) to the group maxima, and each thread
//     keeps the largest key it has seen per query.
// Tensor memory: three accumulator buffers of 128 columns and four A buffers of
// 32 columns.  Every wait is an mbarrier wait with a bound.
//
// With FP8 keys the MMA runs on f16 operands: each query head row (t, j) is
// scaled by a power of two 2^k so that its largest |q| lies in [2^14, 2^15), and
// converted to f16, which is exact for every element down to 2^-32 of that
// maximum (f16 holds bf16's 8 significant bits over that range); the head
// weight is scaled by 2^-k.  Scaling by powers of two commutes with every
// rounding of the fp32 accumulation and of the epilogue, so the scores are
// bit-identical to the bf16 computation whenever the rows' elements are within
// that range; an element below it contributes less than 2^-32 of the row's
// largest term.
//
// First radix pass.  Each (thread, query) pair sees a fixed set of positions
// (its key row of each of the block's tiles); the block histogram of top-12-bit
// bins counts one key per pair, the largest.  Those counts are a lower bound:
// the bin b* where they first reach topk from the top has at least topk keys at
// or above it, i.e. b* <= the bin of the topk-th largest key.  The selection
// then radix-selects among all keys of bin >= b*.  With 148 x 128 pairs per
// query, b* sits near the top 2048 / 18944 of the pair maxima, so for scores
// without heavy ties the candidates number little more than topk.
// ==================================================================================
constexpr int kConvWarps = 4;                // one per TMEM lane quarter
constexpr int kEpiWarps = 12;                // three per lane quarter
constexpr int kEpiPerQuad = kEpiWarps / 4;
constexpr int kIdxWarps = kConvWarps + kEpiWarps + 1;   // and the issuer
constexpr int kIdxThreads = kIdxWarps * 32;
constexpr int kIssuerWarp = kIdxWarps - 1;
constexpr int kQStage = (kMaxT * kHI * 8 + kIdxThreads - 1) / kIdxThreads;   // query chunks staged per thread
constexpr int kRawStagesF8 = 8, kRawStagesBf = 6;
constexpr int kAccBufs = 3, kABufs = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kACol = kAccBufs * 128;   // first column of the A buffers
constexpr int kTileBytesBf16 = kKeyTile * kDI * 2;   // 16 KiB, one 128 x 64 bf16 operand tile
constexpr int kIdxCounters = 16;             // shared words: issue marks
static_assert((kMaxT + kEpiPerQuad - 1) / kEpiPerQuad <= 4, "at most four queries per epilogue warp");
static_assert(kACol + kABufs * 32 <= kTmemCols, "tensor memory budget");
static_assert(kRawStagesF8 <= kBarAFull - kBarRawFull && kRawStagesBf <= kBarSetup - kBarRawEmpty, "mbarrier slots");
static_assert(kRawStagesF8 * kKeyTile * kDI + kTileBytesBf16 + 3 * kMaxT * kHI * 4 + kHistWords * 2 + kIdxCounters * 4 <=
                  kDataBytes,
              "FP8 indexer buffers fit the data region");
static_assert(kRawStagesBf * kTileBytesBf16 + kTileBytesBf16 + 3 * kMaxT * kHI * 4 + kHistWords * 2 + kIdxCounters * 4 <=
                  kDataBytes,
              "bf16 indexer buffers fit the data region");

// Power-of-two exponent k for a query row whose largest |q| has the float bits
// mbits: max * 2^k in [2^14, 2^15); 0 for an all-zero or non-finite row, at most
// 100 (rows below 2^-86 lose low bits).
__device__ __forceinline__ int f16_scale_exp(uint32_t mbits)
{
    const int e = static_cast<int>((mbits >> 23) & 0xFFu) - 127;
    if (mbits == 0u || e == 128) return 0;
    return min(14 - e, 100);
}

__device__ __forceinline__ void red_max_shared(uint32_t* a, uint32_t v)
{
    asm volatile("red.shared::cta.max.u32 [%0], %1;" ::"r"(smem_u32(a)), "r"(v) : "memory");
}

// Everything a warp of the indexer needs.
struct IndexCtx {
    uint8_t* ring;           // [S][raw tile]
    uint8_t* qsw;            // the B operand
    const float* w_s;        // [8][16] head weights
    uint32_t* hs;            // [8][2048] two 16-bit counters per word
    uint32_t* cnt;           // [0] loads issued; [1] MMA groups issued (for the drain after an abort)
    uint32_t* gmax;          // group maxima of the launch, or nullptr
    int64_t gmax_ld;
    uint64_t* raw_full;      // [S] TMA stage landed
    uint64_t* raw_empty;     // [S] (bf16) the stage's MMAs are done
    uint64_t* a_full;        // [4] all four lane quarters of an A buffer written
    uint64_t* a_empty;       // [4] the A buffer's MMAs are done
    uint64_t* acc_full;      // [3] accumulator complete
    uint64_t* acc_empty;     // [3] every epilogue warp has loaded it
    const CUtensorMap* kmap;
    uint64_t policy;
    uint32_t tmem, idesc;
    uint64_t bdesc;
    int nloc;                // tiles of this block
};

template <bool FP8>
struct IndexTile {
    static constexpr int S = FP8 ? kRawStagesF8 : kRawStagesBf;
    static constexpr int kRawBytes = kKeyTile * kDI * (FP8 ? 1 : 2);
    __device__ static int tile_of(int j) { return blockIdx.x + j * static_cast<int>(gridDim.x); }

    // TMA of local tile j into its ring stage (one thread).
    __device__ static void load(const IndexCtx& c, int j)
    {
        const int stage = j % S;
        mbar_arrive_expect_tx(&c.raw_full[stage], kRawBytes);
        tma_load_2d_hint(c.ring + stage * kRawBytes, c.kmap, 0, tile_of(j) * kKeyTile, &c.raw_full[stage], c.policy);
        red_max_shared(&c.cnt[0], static_cast<uint32_t>(j + 1));
    }
    // MMAs of local tile j into accumulator buffer j % 3 (one thread), committed
    // to the buffers they free and fill.
    __device__ static void mma(const IndexCtx& c, int j)
    {
        const uint32_t d = c.tmem + (j % kAccBufs) * 128;
        if constexpr (FP8) {
            const uint32_t a = c.tmem + kACol + (j % kABufs) * 32;
#pragma unroll
            for (int k = 0; k < kDI / 16; ++k) tc_mma_bf16_tmem_a(d, a + k * 8, c.bdesc + 2 * k, c.idesc, k > 0 ? 1u : 0u);
            tc_commit(&c.a_empty[j % kABufs]);
        } else {
            const uint64_t adesc = umma_desc_sw128(smem_u32(c.ring + (j % S) * kRawBytes));
#pragma unroll
            for (int k = 0; k < kDI / 16; ++k) tc_mma_bf16(d, adesc + 2 * k, c.bdesc + 2 * k, c.idesc, k > 0 ? 1u : 0u);
            tc_commit(&c.raw_empty[j % S]);
        }
        tc_commit(&c.acc_full[j % kAccBufs]);
        red_max_shared(&c.cnt[1], static_cast<uint32_t>(j + 1));
    }
};

// Epilogue math of one tile for NQ queries (a compile-time count: straight-line
// code) from the accumulator registers r[u * 16 + j] (query u, head j).  w holds
// half of each head weight: ReLU(x) w = (x + |x|) (w / 2) exactly (x + |x| is 2x
// or +0, both exact; halving w is exact), so each head costs one add (with the
// absolute value as an operand modifier) and half a packed FMA, all on the FMA
// pipe, with the very rounding of fma(max(x, 0), w, acc).  FULL: every key of
// the tile is in range and visible to the warp's queries (no per-key tests).
template <int U0, int N, bool FULL>
__device__ __forceinline__ void index_math(const StepParams& p, const uint32_t (&r)[32], const float* w_half, int s,
                                           float scale, const int (&pos_q)[4], float* const (&out)[4], float (&mx)[4],
                                           uint32_t (&key)[4])
{
    float4 w[N][4];   // half of each head weight (shared memory)
#pragma unroll
    for (int i = 0; i < N; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) w[i][k] = reinterpret_cast<const float4*>(w_half + (U0 + i) * kHI)[k];
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const int u = U0 + i;
        // Four partial sums over heads {j, j+4, j+8, j+12}, j < 4, as two packed fp32
        // FMAs per four heads, combined in a fixed order.
        const float* v = reinterpret_cast<const float*>(&r[i * 16]);
        float2 p01 = make_float2(0.f, 0.f), p23 = make_float2(0.f, 0.f);
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
            const float* x = v + g4 * 4;
            p01 = __ffma2_rn(make_float2(x[0] + fabsf(x[0]), x[1] + fabsf(x[1])), make_float2(w[i][g4].x, w[i][g4].y),
                             p01);
            p23 = __ffma2_rn(make_float2(x[2] + fabsf(x[2]), x[3] + fabsf(x[3])), make_float2(w[i][g4].z, w[i][g4].w),
                             p23);
        }
        const float acc = ((p01.x + p01.y) + (p23.x + p23.y)) * scale;
        key[u] = 0u;
        if (FULL) {
            out[u][s] = acc;
            mx[u] = fmaxf(mx[u], acc);
            key[u] = score_key(acc);
        } else if (s < p.L) {
            const bool vis = s <= pos_q[u];
            out[u][s] = vis ? acc : -INFINITY;
            if (vis) {
                mx[u] = fmaxf(mx[u], acc);
                key[u] = score_key(acc);
            }
        }
    }
}

template <bool FP8>
__device__ void phase_index(const CUtensorMap& kmap, const StepParams& p, uint8_t* smem, uint64_t* bars,
                            uint32_t* tmem_slot)
{
    using Tile = IndexTile<FP8>;
    constexpr int S = Tile::S;
    constexpr int raw_bytes = Tile::kRawBytes;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3;                        // TMEM lane quarter
    const int T = p.T;
    const int ntiles = (visible_max(p) + kKeyTile - 1) / kKeyTile;

    IndexCtx c;
    c.ring = smem;
    c.qsw = smem + S * raw_bytes;
    c.w_s = reinterpret_cast<const float*>(c.qsw + kTileBytesBf16);
    c.hs = reinterpret_cast<uint32_t*>(c.qsw + kTileBytesBf16 + 3 * kMaxT * kHI * 4);   // after weights, halves, exponents
    c.cnt = c.hs + kHistWords / 2;
    c.gmax = p.gmax;
    c.gmax_ld = p.gmax_ld;
    c.raw_full = bars + kBarRawFull;
    c.raw_empty = bars + kBarRawEmpty;
    c.a_full = bars + kBarAFull;
    c.a_empty = bars + kBarAEmpty;
    c.acc_full = bars + kBarAccFull;
    c.acc_empty = bars + kBarAccEmpty;
    c.kmap = &kmap;
    c.policy = l2_evict_first_policy();   // keys are read once; the scores stay in L2
    c.nloc = ntiles > static_cast<int>(blockIdx.x) ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const bool hist = g_view.hist != nullptr;
    uint64_t* setup = bars + kBarSetup;
    float* w_s = const_cast<float*>(c.w_s);

    if (tid == 0) {
        prefetch_tmap(&kmap);
        for (int s = 0; s < S; ++s) {
            mbar_init(&c.raw_full[s], 1);
            if (!FP8) mbar_init(&c.raw_empty[s], 1);
        }
        for (int b = 0; b < kABufs; ++b) {
            mbar_init(&c.a_full[b], kConvWarps);
            mbar_init(&c.a_empty[b], 1);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(&c.acc_full[b], 1);
            mbar_init(&c.acc_empty[b], kEpiWarps);
        }
        mbar_init(setup, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(setup, T * kHI * 4);
        bulk_g2s(w_s, p.w, T * kHI * 4, setup);
    }
    if (tid < kIdxCounters) c.cnt[tid] = 0u;
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    // The indexer queries as the B operand: row r = t*16 + j, 16-byte chunk k at
    // r*128 + (k ^ (r & 7))*16 (the 128B swizzle); rows >= T*16 are never read.
    // FP8 keys: f16 queries, row r scaled by 2^rowk[r] (see above).
    int* rowk = reinterpret_cast<int*>(w_s + 2 * kMaxT * kHI);
    {
        uint4 v[kQStage];   // every load in flight before the first store
#pragma unroll
        for (int u = 0; u < kQStage; ++u) {
            const int i = tid + u * kIdxThreads;
            v[u] = i < T * kHI * 8 ? __ldg(reinterpret_cast<const uint4*>(p.q_idx) + i) : make_uint4(0u, 0u, 0u, 0u);
        }
        if constexpr (FP8) {
            if (tid < kMaxT * kHI) rowk[tid] = 0;   // first the bits of each row's max |q|
            __syncthreads();
#pragma unroll
            for (int u = 0; u < kQStage; ++u) {
                const int i = tid + u * kIdxThreads;
                if (i < T * kHI * 8) {
                    const uint32_t x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    uint32_t m = 0u;
#pragma unroll
                    for (int q = 0; q < 4; ++q) m = max(m, max((x[q] << 16) & 0x7FFFFFFFu, x[q] & 0x7FFF0000u));
                    atomicMax(reinterpret_cast<uint32_t*>(&rowk[i >> 3]), m);   // |q| bits order like |q|
                }
            }
            __syncthreads();
#pragma unroll
            for (int u = 0; u < kQStage; ++u) {
                const int i = tid + u * kIdxThreads, r = i >> 3, k = i & 7;
                if (i < T * kHI * 8) {
                    const float sc = __int_as_float((127 + f16_scale_exp(static_cast<uint32_t>(rowk[r]))) << 23);
                    const uint32_t x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    uint32_t y[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const __half2 h = __floats2half2_rn(__uint_as_float(x[q] << 16) * sc,
                                                            __uint_as_float(x[q] & 0xFFFF0000u) * sc);
                        y[q] = *reinterpret_cast<const uint32_t*>(&h);
                    }
                    *reinterpret_cast<uint4*>(c.qsw + r * 128 + ((k ^ (r & 7)) << 4)) = make_uint4(y[0], y[1], y[2], y[3]);
                }
            }
            __syncthreads();
            if (tid < kMaxT * kHI) rowk[tid] = f16_scale_exp(static_cast<uint32_t>(rowk[tid]));
        } else {
#pragma unroll
            for (int u = 0; u < kQStage; ++u) {
                const int i = tid + u * kIdxThreads, r = i >> 3, k = i & 7;
                if (i < T * kHI * 8) *reinterpret_cast<uint4*>(c.qsw + r * 128 + ((k ^ (r & 7)) << 4)) = v[u];
            }
        }
    }
    if (hist)
        for (int i = tid; i < kHistWords / 2; i += kIdxThreads) c.hs[i] = 0u;
    fence_proxy_async_smem();   // the queries are read by the tensor cores (async proxy)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    c.tmem = *tmem_slot;
    c.idesc = FP8 ? umma_idesc_f16(kKeyTile, T * kHI) : umma_idesc_bf16(kKeyTile, T * kHI);
    c.bdesc = umma_desc_sw128(smem_u32(c.qsw));
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int row = quad * 32 + lane;                // this thread's key row of every tile
    if (tid == 0)
        for (int j = 0; j < S && j < c.nloc; ++j) Tile::load(c, j);
    bool aborted = __any_sync(0xffffffffu, !mbar_wait(setup, 0, p.err));   // warp-uniform from here on
    // half of every head weight, next to the weights (see index_math)
    float* w_half = w_s + kMaxT * kHI;
    if (tid < T * kHI) w_half[tid] = 0.5f * w_s[tid] * (FP8 ? __int_as_float((127 - rowk[tid]) << 23) : 1.0f);
    __syncthreads();

    // per-thread key maxima of the epilogue warps' queries (NaN: none yet)
    float mx[4] = {NAN, NAN, NAN, NAN};
    const bool epi = warp >= kConvWarps && warp < kConvWarps + kEpiWarps;
    const int e_idx = epi ? (warp - kConvWarps) / 4 : 0;
    const int qa = e_idx * T / kEpiPerQuad;
    const int nq = epi ? (e_idx + 1) * T / kEpiPerQuad - qa : 0;   // 0..4

    if (warp < kConvWarps) {
        // ---------------- converter / issuer warps ----------------
        if constexpr (FP8) {
            for (int j = 0; j < c.nloc && !aborted; ++j) {
                const int ab = j % kABufs, stage = j % S;
                bool ok = j < kABufs || mbar_wait(&c.a_empty[ab], ((j / kABufs) - 1) & 1, p.err);
                ok = ok && mbar_wait(&c.raw_full[stage], (j / S) & 1, p.err);
                if (__any_sync(0xffffffffu, !ok)) {
                    aborted = true;
                    break;
                }
                // row `row`: 64 codes, 16-byte chunk q stored at chunk q ^ ((row >> 1) & 3)
                const uint8_t* src = c.ring + stage * raw_bytes + row * 64;
                uint4 v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) v[q] = *reinterpret_cast<const uint4*>(src + ((q ^ ((row >> 1) & 3)) << 4));
                uint32_t r[32];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t x[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        r[8 * q + 2 * h] = e4m3x2_to_f16x2(x[h]);
                        r[8 * q + 2 * h + 1] = e4m3x2_to_f16x2(x[h] >> 16);
                    }
                }
                tmem_st32(c.tmem + lane_base + kACol + ab * 32, r);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&c.a_full[ab]);
            }
        }
    } else if (warp == kIssuerWarp) {
        // ---------------- the issuer: one thread issues every tile's MMAs ----------------
        // once its A operand is in (FP8: all four lane quarters widened; bf16: the TMA
        // tile landed) and its accumulator buffer is free, and refills the ring: FP8,
        // tile j's stage (every converter has read it) with tile j + S; bf16, the stage
        // two tiles behind once its MMAs are done.
        bool ok = !aborted;
        if (lane == 0 && ok) {
            for (int j = 0; j < c.nloc && ok; ++j) {
                if constexpr (FP8) ok = mbar_wait(&c.a_full[j % kABufs], (j / kABufs) & 1, p.err);
                else ok = mbar_wait(&c.raw_full[j % S], (j / S) & 1, p.err);
                ok = ok && (j < kAccBufs || mbar_wait(&c.acc_empty[j % kAccBufs], ((j / kAccBufs) - 1) & 1, p.err));
                if (!ok) break;
                tc_fence_after();
                Tile::mma(c, j);
                if constexpr (FP8) {
                    if (j + S < c.nloc) Tile::load(c, j + S);
                } else {
                    const int f = j - 2;
                    if (f >= 0 && f + S < c.nloc) {
                        ok = mbar_wait(&c.raw_empty[f % S], (f / S) & 1, p.err);
                        if (ok) Tile::load(c, f + S);
                    }
                }
            }
        }
        aborted = __any_sync(0xffffffffu, !ok);
    } else {
        // ---------------- epilogue warps ----------------
        const float* wq = w_half + qa * kHI;         // this warp's queries' halved weights
        int pos_q[4];                                // positions of this warp's queries
        float* out[4];                               // their score rows
        int pos_min = p.L;                           // tiles wholly below it and below L need no tests
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            pos_q[u] = u < nq ? query_pos_rt(p, qa + u) : -1;
            out[u] = p.scores + (int64_t)min(qa + u, T - 1) * p.ld;
            if (u < nq) pos_min = min(pos_min, pos_q[u] + 1);
        }
        auto run = [&](auto nq_tag) {
            constexpr int NQ = decltype(nq_tag)::value;
            const bool scaled = p.scale != nullptr;
            float scale_next = 1.0f;
            if (NQ > 0 && scaled && c.nloc > 0) {
                const int s = Tile::tile_of(0) * kKeyTile + row;
                scale_next = s < p.L ? __ldg(p.scale + s) : 1.0f;
            }
            for (int e = 0; e < c.nloc && !aborted; ++e) {
                const int tile = Tile::tile_of(e);
                const int s = tile * kKeyTile + row;
                const float scale = scale_next;
                if (NQ > 0 && scaled && e + 1 < c.nloc) {   // next tile's scale, in flight during this tile
                    const int s2 = Tile::tile_of(e + 1) * kKeyTile + row;
                    scale_next = s2 < p.L ? __ldg(p.scale + s2) : 1.0f;
                }
                const int cb = e % kAccBufs;
                if (__any_sync(0xffffffffu, !mbar_wait(&c.acc_full[cb], (e / kAccBufs) & 1, p.err))) {
                    aborted = true;
                    break;
                }
                tc_fence_after();
                // queries in groups of two: one 32-column load, then its math; the buffer is
                // released after the last load, while the last group's math runs
                const uint32_t tbase = c.tmem + lane_base + cb * 128 + qa * kHI;
                const bool full = tile * kKeyTile + kKeyTile <= pos_min;
                uint32_t key[4] = {0u, 0u, 0u, 0u};
                auto group = [&](auto g_tag) {
                    constexpr int G = decltype(g_tag)::value;             // queries [2G, 2G + n)
                    constexpr int n = NQ - 2 * G >= 2 ? 2 : NQ - 2 * G;
                    uint32_t r[32];
                    if constexpr (n == 1) tmem_ld16_nowait(tbase + 32 * G, reinterpret_cast<uint32_t(&)[16]>(r[0]));
                    else tmem_ld32_nowait(tbase + 32 * G, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < n * 16; ++k) asm volatile("" : "+r"(r[k]));   // no use before the wait
                    if (2 * G + n >= NQ) {   // the last load of this buffer
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&c.acc_empty[cb]);
                    }
                    if (full) index_math<2 * G, n, true>(p, r, wq, s, scale, pos_q, out, mx, key);
                    else index_math<2 * G, n, false>(p, r, wq, s, scale, pos_q, out, mx, key);
                };
                if constexpr (NQ == 0) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&c.acc_empty[cb]);
                } else {
                    group(std::integral_constant<int, 0>{});
                    if constexpr (NQ > 2) group(std::integral_constant<int, 1>{});
                }
                if constexpr (NQ > 0) {
                    if (c.gmax != nullptr) {
                        // the largest key of this warp's 32 positions per query (lane u stores
                        // query u's): lets the extraction skip groups below its cut
                        uint32_t mine = 0u;
#pragma unroll
                        for (int u = 0; u < NQ; ++u) {
                            const uint32_t m = __reduce_max_sync(0xffffffffu, key[u]);
                            if (lane == u) mine = m;
                        }
                        if (lane < NQ)
                            c.gmax[(int64_t)(qa + lane) * c.gmax_ld + tile * (kKeyTile / 32) + quad] = mine;
                    }
                }
            }
        };
        if (nq == 4) {
            run(std::integral_constant<int, 4>{});
        } else if (nq == 3) {
            run(std::integral_constant<int, 3>{});
        } else if (nq == 2) {
            run(std::integral_constant<int, 2>{});
        } else if (nq == 1) {
            run(std::integral_constant<int, 1>{});
        } else {
            run(std::integral_constant<int, 0>{});
        }
    }
    // A wait that ran out (error bit set) ends the loop for that warp; the others
    // run into bounded waits and stop too.  Copies and MMAs still in flight land
    // before the shared memory and tensor memory are reused: the last S loads and
    // the last three MMA groups.
    aborted = __syncthreads_or(aborted);
    if (aborted) {
        if (tid == 0) {
            const int li = static_cast<int>(c.cnt[0]);
            for (int k = max(0, li - S); k < li; ++k) mbar_wait(&c.raw_full[k % S], (k / S) & 1, p.err);
        }
        if (tid == 32) {
            const int mi = static_cast<int>(c.cnt[1]);
            for (int k = max(0, mi - kAccBufs); k < mi; ++k)
                mbar_wait(&c.acc_full[k % kAccBufs], (k / kAccBufs) & 1, p.err);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(c.tmem, kTmemCols);
    }
    if (hist) {
        // one count per (thread, query): its largest key's bin
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (u < nq && !isnan(mx[u])) {
                const uint32_t k = score_key(mx[u]);
                atomicAdd(&c.hs[(qa + u) * (kHistBins / 2) + (k >> (kHistShift + 1))], 1u << (((k >> kHistShift) & 1u) << 4));
            }
        __syncthreads();
        // the block's 16-bit counters (two per word) into the launch's histogram
        for (int i = tid; i < T * (kHistBins / 2); i += kIdxThreads) {
            const uint32_t v = c.hs[i];
            if (v) {
                uint32_t* gh = g_view.hist + (i / (kHistBins / 2)) * kHistBins + 2 * (i % (kHistBins / 2));
                if (v & 0xFFFFu) atomicAdd(gh, v & 0xFFFFu);
                if (v >> 16) atomicAdd(gh + 1, v >> 16);
            }
        }
    }
    // Positions no query can see (s >= n_max): -inf, as the stage contract states.
    const int64_t tail0 = (int64_t)ntiles * kKeyTile;
    for (int64_t s = tail0 + (int64_t)blockIdx.x * kIdxThreads + tid; s < p.L; s += (int64_t)gridDim.x * kIdxThreads)
        for (int tt = 0; tt < T; ++tt) p.scores[(int64_t)tt * p.ld + s] = -INFINITY;
}

// Phase 1 for caller-provided scores: the histogram of their keys' top 12 bits,
// each block over a slice of every query's visible positions.  A NaN score is
// invalid input and flags the top-k error bit.
__device__ void phase_hist_scores(const StepParams& p, uint8_t* smem)
{
    uint32_t* h = reinterpret_cast<uint32_t*>(smem);   // [kHistBins]
    const int tid = threadIdx.x;
    const int64_t per = ((visible_max(p) + (int64_t)gridDim.x - 1) / gridDim.x + 3) / 4 * 4;
    for (int t = 0; t < p.T; ++t) {
        const int n = query_pos_rt(p, t) + 1;
        if (n <= p.topk) continue;
        for (int b = tid; b < kHistBins; b += kThreads) h[b] = 0u;
        __syncthreads();
        // this block's slice [s0, s1): s0 is a multiple of 4 unless the slice is empty
        const int64_t s0 = (int64_t)blockIdx.x * per, s1 = min((int64_t)n, s0 + per);
        const float4* row = reinterpret_cast<const float4*>(p.scores + (int64_t)t * p.ld);
        bool nan = false;
        for (int64_t q0 = s0 / 4; q0 * 4 < s1; q0 += 4 * kThreads) {
            float4 v[4];   // four loads in flight per thread
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t q = q0 + u * kThreads + tid;
                v[u] = q * 4 < s1 ? __ldcg(row + q) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t s = (q0 + u * kThreads + tid) * 4;
                const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (s + k >= s0 && s + k < s1) {
                        nan |= f[k] != f[k];
                        atomicAdd(&h[score_key(f[k]) >> kHistShift], 1u);
                    }
            }
        }
        if (nan) atomicOr(p.err, ERR_TOPK_STATE);
        __syncthreads();
        for (int b = tid; b < kHistBins; b += kThreads)
            if (h[b]) atomicAdd(g_view.hist + t * kHistBins + b, h[b]);
        __syncthreads();
    }
}

// ==================================================================================
// Phase 2: candidate extraction, one item per (query t, chunk c) and block.
// The query's cut bin comes from the launch's histogram: the threshold bin b*
// (the bin of its topk-th largest key) for an exact histogram, a bin at or below
// it for the indexer's lower-bound one; every visible key in the cut bin or
// above is a candidate.  Warp w of the block takes its own eighth of the chunk:
// with group maxima it reads only the scores of the 32-position groups whose
// maximum reaches the cut, else it streams its scores through a private ring of
// 4 KiB bulk copies; it appends its candidates, in position order, to its
// sub-segment of the query's list (which starts at the sub-range's first
// position, so it can never overflow).  No block-wide barrier in the loop.
// ==================================================================================
constexpr int kXStages = 4;
constexpr int kXPiece = 1024;                 // scores per bulk copy
constexpr int kXHistOff = kWarps * kXStages * kXPiece * 4;   // the histogram copy, after the rings
static_assert(kXHistOff + kHistBins * 4 <= kDataBytes, "extraction buffers fit");

__device__ void phase_extract(const StepParams& p, uint8_t* smem, uint64_t* bars, uint32_t* res, uint32_t* scratch)
{
    const int i = blockIdx.x;
    if (i >= p.T * p.nchunk) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t = i / p.nchunk, c = i % p.nchunk;
    const int n = query_pos_rt(p, t) + 1;
    uint64_t* full = bars + kBarExtract + warp * kXStages;
    if (n > p.topk) {
        const bool bound = p.hist_bound != 0;
        const int R = p.chunk / kSegPerChunk;
        const int s0 = c * p.chunk + warp * R, s1 = min(s0 + R, n);
        // With group maxima: their first round is loaded now, in flight while the
        // cut is found (they do not depend on it).
        const bool use_gmax = p.gmax != nullptr && bound;
        const uint32_t* gm = p.gmax + (int64_t)t * p.gmax_ld;
        uint32_t m_first[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int g = s0 + (k * 32 + lane) * 32;
            m_first[k] = use_gmax && g < s1 ? __ldcg(gm + g / 32) : 0u;
        }
        // threshold bin from the histogram (coalesced loads, all in flight)
        uint32_t* h = reinterpret_cast<uint32_t*>(smem + kXHistOff);
        {
            uint32_t v[kHistBins / kThreads];
#pragma unroll
            for (int k = 0; k < kHistBins / kThreads; ++k)
                v[k] = __ldcg(g_view.hist + t * kHistBins + tid + k * kThreads);
#pragma unroll
            for (int k = 0; k < kHistBins / kThreads; ++k) h[tid + k * kThreads] = v[k];
        }
        if (lane == 0)
            for (int s = 0; s < kXStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
        fence_proxy_async_smem();   // earlier generic writes to the ring region come first
        __syncthreads();
        find_from_top(h, static_cast<uint32_t>(p.topk), res);
        // Exact histogram (caller scores): the candidates are the keys of the threshold
        // bin and above, those above it all selected.  Indexer histogram of per-thread
        // maxima (a lower bound): every key of bin >= b* is a candidate, to be
        // radix-selected from the top; with fewer than topk counts, every visible key.
        uint32_t cut = 0u, above = 0u, top = 0xFFFFFFFFu;
        if (res[2]) {
            cut = res[0] << kHistShift;
            if (!bound) {
                above = res[1];
                top = bin_top(cut, kHistShift, 0xFFFFFFFFu);
            }
        } else if (!bound && tid == 0) {   // histogram and scores disagree: cannot happen for consistent input
            atomicOr(p.err, ERR_TOPK_STATE);
        }
        if (c == 0 && tid == 0) reinterpret_cast<uint4*>(p.cuts)[t] = make_uint4(cut, above, top, 0u);

        const int np = s1 > s0 ? (s1 - s0 + kXPiece - 1) / kXPiece : 0;
        const float* row = p.scores + (int64_t)t * p.ld;
        float* ring = reinterpret_cast<float*>(smem) + warp * kXStages * kXPiece;
        uint2* out = p.list + (int64_t)t * p.list_ld + s0;
        uint32_t count = 0;
        if (use_gmax) {
            // Only the 32-position groups whose largest key reaches the cut are read:
            // eight rounds of 32 group maxima in flight per lane; the hit groups of all
            // eight go to a short list in position order (in this warp's ring, idle
            // here), then their scores are read eight groups at a time.
            uint16_t* hl = reinterpret_cast<uint16_t*>(ring);   // group index within the round
            for (int base = s0; base < s1; base += 8 * 32 * 32) {
                uint32_t m[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int g = base + (k * 32 + lane) * 32;
                    m[k] = base == s0 ? m_first[k] : (g < s1 ? __ldcg(gm + g / 32) : 0u);
                }
                int nh = 0;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const bool h = base + (k * 32 + lane) * 32 < s1 && m[k] >= cut;
                    const uint32_t hm = __ballot_sync(0xffffffffu, h);
                    if (h) hl[nh + __popc(hm & ((1u << lane) - 1u))] = static_cast<uint16_t>(k * 32 + lane);
                    nh += __popc(hm);
                }
                __syncwarp();
                for (int j = 0; j < nh; j += 8) {
                    int sp[8];
                    float f[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        sp[u] = j + u < nh ? base + static_cast<int>(hl[j + u]) * 32 + lane : s1;
                        f[u] = sp[u] < s1 ? __ldcg(row + sp[u]) : -INFINITY;
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        if (j + u < nh) {
                            const uint32_t key = score_key(f[u]);
                            const bool take = sp[u] < s1 && key >= cut;
                            const uint32_t tb = __ballot_sync(0xffffffffu, take);
                            if (take) out[count + __popc(tb & ((1u << lane) - 1u))] = make_uint2(key, static_cast<uint32_t>(sp[u]));
                            count += __popc(tb);
                        }
                    }
                }
                __syncwarp();   // the list is rewritten by the next round
            }
        } else {
            auto issue = [&](int j) {
                const int a = s0 + j * kXPiece;
                const uint32_t bytes = static_cast<uint32_t>((min(kXPiece, s1 - a) + 3) & ~3) * 4u;
                mbar_arrive_expect_tx(&full[j % kXStages], bytes);
                bulk_g2s(ring + (j % kXStages) * kXPiece, row + a, bytes, &full[j % kXStages]);
            };
            if (lane == 0)
                for (int j = 0; j < min(np, kXStages); ++j) issue(j);
            int j = 0;
            for (; j < np; ++j) {
                if (__any_sync(0xffffffffu, !mbar_wait(&full[j % kXStages], (j / kXStages) & 1, p.err))) break;
                const float* buf = ring + (j % kXStages) * kXPiece;
                const int a = s0 + j * kXPiece;
#pragma unroll 2
                for (int k = 0; k < kXPiece / 128; ++k) {
                    const int base = a + k * 128 + lane * 4;
                    const float4 f = *reinterpret_cast<const float4*>(buf + k * 128 + lane * 4);
                    const uint32_t key[4] = {score_key(f.x), score_key(f.y), score_key(f.z), score_key(f.w)};
                    uint32_t m = 0;
#pragma unroll
                    for (int q = 0; q < 4; ++q) m |= static_cast<uint32_t>(base + q < s1 && key[q] >= cut) << q;
                    if (__ballot_sync(0xffffffffu, m != 0u)) {
                        const uint32_t my = __popc(m);
                        const uint32_t incl = warp_incl_scan(my);
                        uint32_t o = count + incl - my;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            if (m & (1u << q)) out[o++] = make_uint2(key[q], static_cast<uint32_t>(base + q));
                        count += __shfl_sync(0xffffffffu, incl, 31);
                    }
                }
                __syncwarp();
                if (lane == 0 && j + kXStages < np) issue(j + kXStages);
            }
            if (j < np && lane == 0)   // a wait ran out: let the copies in flight land
                for (int k = j; k < min(np, j + kXStages); ++k) mbar_wait(&full[k % kXStages], (k / kXStages) & 1, p.err);
        }
        if (lane == 0) p.seg_n[t * kMaxSeg + c * kSegPerChunk + warp] = count;
    }
    __syncthreads();
    if (tid == 0) red_release_add(p.ctrl + kCtrlWordArrive + t, 1u);
}

// Candidates held in registers by the selection: up to kSelReg per thread, a
// contiguous run of the position-ordered list each.
constexpr int kSelReg = 16;

// One radix pass over the keys in registers (k[u], u < cnt, of every thread):
// the bin of [lo, hi] (at most 4096 bins of width 2^shift) holding the need-th
// largest key becomes the new [lo, hi]; need drops by the keys above that bin.
// Thread i sums bins [4096 - 16 (i + 1), 4096 - 16 i), so one block-wide scan
// in thread order counts from the top; the thread whose run holds the need-th
// key finds the bin within its 16.
__device__ void radix_pass_reg(const uint32_t (&k)[kSelReg], int cnt, uint32_t& lo, uint32_t& hi, uint32_t& need,
                               uint32_t* h, uint32_t* res, uint32_t* scratch, uint32_t* err)
{
    static_assert(kHistBins == 16 * kThreads, "16 bins per thread");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // Narrow [lo, hi] to the keys actually in it first: candidate keys cluster in a
    // few bins of a wide range, and same-address shared atomics serialise.
    {
        uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
        for (int u = 0; u < kSelReg; ++u)
            if (u < cnt && k[u] >= lo && k[u] <= hi) {
                mn = min(mn, k[u]);
                mx = max(mx, k[u]);
            }
        mn = __reduce_min_sync(0xffffffffu, mn);
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (lane == 0) {
            scratch[32 + warp] = mn;
            scratch[48 + warp] = mx;
        }
        __syncthreads();
        mn = 0xFFFFFFFFu;
        mx = 0u;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            mn = min(mn, scratch[32 + w]);
            mx = max(mx, scratch[48 + w]);
        }
        if (mn <= mx) {   // else no key in range: the search below reports it
            lo = mn;
            hi = mx;
        }
    }
    const int shift = range_shift(lo, hi);
    for (int i = tid; i < kHistBins / 4; i += kThreads) reinterpret_cast<uint4*>(h)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (tid == 0) res[2] = 0u;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kSelReg; ++u)
        if (u < cnt && k[u] >= lo && k[u] <= hi) atomicAdd(&h[(k[u] - lo) >> shift], 1u);
    __syncthreads();
    const int b0 = kHistBins - 16 * (tid + 1);
    uint32_t c[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 v = reinterpret_cast<const uint4*>(h + b0)[q];
        c[4 * q] = v.x;
        c[4 * q + 1] = v.y;
        c[4 * q + 2] = v.z;
        c[4 * q + 3] = v.w;
    }
    uint32_t sum = 0;
#pragma unroll
    for (int q = 0; q < 16; ++q) sum += c[q];
    uint32_t total;
    const uint32_t before = block_excl_scan(sum, total, scratch);   // keys in the bins above this thread's
    if (before < need && before + sum >= need) {
        uint32_t run = before;
        int bin = -1;
        uint32_t above = 0;
#pragma unroll
        for (int q = 15; q >= 0; --q) {
            if (bin < 0 && run + c[q] >= need) {
                bin = b0 + q;
                above = run;
            }
            run += c[q];
        }
        res[0] = static_cast<uint32_t>(bin);
        res[1] = above;
        res[2] = 1u;
    }
    __syncthreads();
    if (!res[2]) {   // fewer keys in [lo, hi] than needed: inconsistent candidates
        if (tid == 0) atomicOr(err, ERR_TOPK_STATE);
        __syncthreads();
        if (tid == 0) {
            res[0] = 0u;
            res[1] = 0u;
        }
        __syncthreads();
    }
    const uint32_t nlo = lo + (res[0] << shift);
    const uint32_t nhi = bin_top(nlo, shift, hi);
    need -= res[1];
    lo = nlo;
    hi = nhi;
    // A bin of at most 256 keys is resolved at once instead of by another pass: its
    // keys go to a short list, and thread i ranks key i against the list (every
    // thread reads the same entry at a time: broadcasts); the key with (keys above
    // it) < need <= (keys at or above it) is the exact one.
    const uint32_t in_bin = h[res[0]];
    __syncthreads();
    if (shift > 0 && in_bin <= static_cast<uint32_t>(kThreads) && res[2]) {
        uint32_t* list = h;   // the bins are no longer needed
        if (tid == 0) {
            res[1] = 0u;   // list length
            res[2] = 0u;   // becomes the ties to take, once found
        }
        __syncthreads();
        {   // one shared atomic per warp: a warp scan places each thread's keys
            uint32_t c = 0;
#pragma unroll
            for (int u = 0; u < kSelReg; ++u) c += u < cnt && k[u] >= nlo && k[u] <= nhi;
            const uint32_t incl = warp_incl_scan(c);
            uint32_t base = 0;
            if (lane == 31 && incl) base = atomicAdd(&res[1], incl);
            uint32_t o = __shfl_sync(0xffffffffu, base, 31) + incl - c;
#pragma unroll
            for (int u = 0; u < kSelReg; ++u)
                if (u < cnt && k[u] >= nlo && k[u] <= nhi) list[o++] = k[u];
        }
        __syncthreads();
        const uint32_t n = res[1];
        const uint32_t mine = tid < static_cast<int>(n) ? list[tid] : 0u;
        // four list entries per shared load (a broadcast); the entries past n are masked
        uint32_t gt = 0, ge = 0;
        if (warp * 32 < static_cast<int>(n)) {
            const uint4* l4 = reinterpret_cast<const uint4*>(list);
#pragma unroll 2
            for (uint32_t j = 0; j < n; j += 4) {
                const uint4 o = l4[j / 4];
                const uint32_t e[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (j + q < n) {
                        gt += e[q] > mine;
                        ge += e[q] >= mine;
                    }
            }
        }
        // every holder of the exact key finds it; they agree on (key, need - gt)
        if (tid < static_cast<int>(n) && gt < need && need <= ge) {
            res[0] = mine;
            res[2] = need - gt;
        }
        __syncthreads();
        if (res[2]) {
            lo = hi = res[0];
            need = res[2];
        } else if (tid == 0) {
            atomicOr(err, ERR_TOPK_STATE);
        }
    }
    __syncthreads();
}

// ==================================================================================
// Phase 3: the selection of query t, by block t once every extraction item of
// the query is done.  The candidates (every key in the cut bin or above,
// position-ordered sub-segments) are gathered into shared memory in order; a
// radix select from the top of their key range finds tau, the topk-th
// largest key, and how many keys equal to tau are taken (the lowest positions,
// i.e. the first ones in list order); an ordered compaction writes the
// selected positions ascending.  More candidates than fit in shared memory
// (heavy ties) take the same steps over the list in global memory.
// ==================================================================================
constexpr int kSelHOff = 0;                              // [kHistBins] select bins
constexpr int kSelOffOff = kHistBins * 4;                // [kMaxSeg] sub-segment offsets
constexpr int kSelEntOff = kSelOffOff + kMaxSeg * 4;     // candidates (key, position)
constexpr int kSelCap = (kDataBytes - kSelEntOff) / 10 / 256 * 256;   // with a 16-bit sub-segment index each
constexpr int kSelSegOff = kSelEntOff + kSelCap * 8;     // [kSelCap] sub-segment of each candidate
constexpr int kSelGOff = kSelEntOff + kMaxSeg * 4;       // (global path) second per-sub-segment array
constexpr int kSelPieceOff = kSelEntOff + 2 * kSelReg * kThreads * 4;   // (register path) [kMaxSeg] first piece
static_assert(kSelPieceOff + kMaxSeg * 4 <= kDataBytes, "piece numbers fit");
static_assert(kSelCap >= 4096 && kSelSegOff + kSelCap * 2 <= kDataBytes && kSelGOff + kMaxSeg * 4 <= kDataBytes,
              "selection buffers fit");
static_assert(kMaxSeg <= 65536, "sub-segment indices fit 16 bits");

__device__ __forceinline__ int seg_start(const StepParams& p, int i)
{
    return (i / kSegPerChunk) * p.chunk + (i % kSegPerChunk) * (p.chunk / kSegPerChunk);
}

__device__ void phase_select(const StepParams& p, uint8_t* smem, uint32_t* res, uint32_t* scratch, int* ok_s)
{
    const int t = blockIdx.x;
    if (t >= p.T) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = query_pos_rt(p, t) + 1;
    const uint32_t topk = static_cast<uint32_t>(p.topk);
    int32_t* sel = p.sel + (int64_t)t * p.sel_ld;
    if (n <= p.topk) {   // everything visible is selected
        for (int j = tid; j < p.topk; j += kThreads) sel[j] = j < n ? j : -1;
    } else {
        if (tid == 0) *ok_s = wait_counter(p, p.ctrl + kCtrlWordArrive + t, static_cast<uint32_t>(p.nchunk)) ? 1 : 0;
        __syncthreads();
        stamp(p, 4);
        if (*ok_s) {
            uint32_t* h = reinterpret_cast<uint32_t*>(smem + kSelHOff);
            uint32_t* off = reinterpret_cast<uint32_t*>(smem + kSelOffOff);
            const int nseg = p.nchunk * kSegPerChunk;
            const uint32_t* segn = p.seg_n + t * kMaxSeg;
            for (int k = tid; k < nseg; k += kThreads) off[k] = __ldcg(segn + k);
            const uint4 cq = __ldcg(reinterpret_cast<const uint4*>(p.cuts) + t);
            __syncthreads();
            const uint32_t m = block_scan_array(off, nseg, scratch);   // off[k]: first slot of sub-segment k
            uint32_t lo = cq.x, hi = cq.z;   // the keys of [lo, hi] are radix-selected
            uint32_t need = topk - cq.y;     // keys above hi are all taken
            const uint2* glist = p.list + (int64_t)t * p.list_ld;
            auto seg_cnt = [&](int k) { return (k + 1 < nseg ? off[k + 1] : m) - off[k]; };
            uint32_t nsel = 0;
            if (m <= static_cast<uint32_t>(kSelReg * kThreads)) {
                // ---- few candidates: a run of up to 16 per thread, in registers ----
                // The list into shared memory in list order, in pieces of 16 entries: a scan
                // of the sub-segments' piece counts numbers the pieces, thread i takes pieces
                // i and i + 256 (a binary search finds each one's sub-segment), all loads in
                // flight; then thread i takes entries [i per, (i + 1) per).  (Loading each
                // thread's run straight into registers is slower: every warp load then
                // touches 32 scattered sectors.)
                uint32_t* ckey = reinterpret_cast<uint32_t*>(smem + kSelEntOff);
                uint32_t* cpos = ckey + kSelReg * kThreads;
                uint32_t* cpre = reinterpret_cast<uint32_t*>(smem + kSelPieceOff);
                for (int k = tid; k < nseg; k += kThreads) cpre[k] = (seg_cnt(k) + 15u) / 16u;
                __syncthreads();
                const uint32_t npiece = block_scan_array(cpre, nseg, scratch);   // cpre[k]: first piece of k
                for (uint32_t q0 = tid; q0 < npiece; q0 += 2 * kThreads) {
                    uint4 v[2][8];
                    uint32_t jj[2], cc[2], oo[2];
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const uint32_t q = q0 + h2 * kThreads;
                        int k = 0;   // the last sub-segment with cpre[k] <= q: a non-empty one
                        for (int step = 1 << (31 - __clz(nseg)); step > 0; step >>= 1)
                            if (k + step < nseg && cpre[k + step] <= q) k += step;
                        const bool any = q < npiece;
                        jj[h2] = any ? (q - cpre[k]) * 16u : 0u;
                        cc[h2] = any ? seg_cnt(k) : 0u;
                        oo[h2] = off[k];
                        const uint4* src = reinterpret_cast<const uint4*>(glist + seg_start(p, k)) + jj[h2] / 2;
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            v[h2][u] = jj[h2] + 2 * u < cc[h2] ? __ldcg(src + u) : make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const uint32_t e = jj[h2] + 2 * u, o = oo[h2];
                            if (e < cc[h2]) {
                                ckey[o + e] = v[h2][u].x;
                                cpos[o + e] = v[h2][u].y;
                            }
                            if (e + 1 < cc[h2]) {
                                ckey[o + e + 1] = v[h2][u].z;
                                cpos[o + e + 1] = v[h2][u].w;
                            }
                        }
                }
                __syncthreads();
                const uint32_t per = (m + kThreads - 1) / kThreads;
                const uint32_t j0 = min(m, tid * per), j1 = min(m, j0 + per);
                const int cnt = static_cast<int>(j1 - j0);
                uint32_t key[kSelReg], pos[kSelReg];
#pragma unroll
                for (int u = 0; u < kSelReg; ++u) {
                    key[u] = u < cnt ? ckey[j0 + u] : 0u;
                    pos[u] = u < cnt ? cpos[j0 + u] : 0u;
                }
#pragma unroll 1
                for (int pass = 0; pass < 4 && lo != hi; ++pass)
                    radix_pass_reg(key, cnt, lo, hi, need, h, res, scratch, p.err);
                const uint32_t tau = lo;
                // ordered compaction: one block scan of (keys above tau, ties) counts, packed
                // as 16 + 16 bits (m <= 4096); ties are taken lowest position first
                uint32_t gt = 0, eq = 0;
#pragma unroll
                for (int u = 0; u < kSelReg; ++u)
                    if (u < cnt) {
                        gt += key[u] > tau;
                        eq += key[u] == tau;
                    }
                uint32_t tot;
                const uint32_t ex = block_excl_scan((gt << 16) | eq, tot, scratch);
                uint32_t tie = ex & 0xFFFFu;
                uint32_t o = (ex >> 16) + min(tie, need);
                nsel = (tot >> 16) + min(tot & 0xFFFFu, need);
#pragma unroll
                for (int u = 0; u < kSelReg; ++u)
                    if (u < cnt) {
                        const bool eqk = key[u] == tau;
                        if (key[u] > tau || (eqk && tie < need)) {
                            if (o < topk) sel[o] = static_cast<int32_t>(pos[u]);
                            ++o;
                        }
                        tie += eqk;
                    }
            } else if (m <= static_cast<uint32_t>(kSelCap)) {
                // ---- the candidates fit in shared memory ----
                // Entry j's sub-segment: every non-empty sub-segment writes its index at its
                // first slot, then a running maximum fills the slots in between.  The loads
                // are then independent: eight in flight per thread.
                uint2* ent = reinterpret_cast<uint2*>(smem + kSelEntOff);
                uint16_t* segof = reinterpret_cast<uint16_t*>(smem + kSelSegOff);
                for (uint32_t j = tid; j < m; j += kThreads) segof[j] = 0;
                __syncthreads();
                for (int k = tid; k < nseg; k += kThreads)
                    if (seg_cnt(k)) segof[off[k]] = static_cast<uint16_t>(k);
                __syncthreads();
                {
                    const uint32_t per = (m + kThreads - 1) / kThreads;
                    const uint32_t j0 = min(m, tid * per), j1 = min(m, j0 + per);
                    uint32_t run = 0;
                    for (uint32_t j = j0; j < j1; ++j) run = max(run, static_cast<uint32_t>(segof[j]));
                    const uint32_t before = block_excl_max(run, scratch);
                    run = before;
                    for (uint32_t j = j0; j < j1; ++j) {
                        run = max(run, static_cast<uint32_t>(segof[j]));
                        segof[j] = static_cast<uint16_t>(run);
                    }
                }
                __syncthreads();
                for (uint32_t j0 = 0; j0 < m; j0 += 8 * kThreads) {
                    uint2 v[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const uint32_t j = j0 + u * kThreads + tid;
                        v[u] = make_uint2(0u, 0u);
                        if (j < m) {
                            const int k = segof[j];
                            v[u] = __ldcg(glist + seg_start(p, k) + (j - off[k]));
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const uint32_t j = j0 + u * kThreads + tid;
                        if (j < m) ent[j] = v[u];
                    }
                }
                __syncthreads();
#pragma unroll 1
                for (int pass = 0; pass < 4 && lo != hi; ++pass)
                    radix_pass(
                        [&](auto add) {
                            for (uint32_t j = tid; j < m; j += kThreads) add(ent[j].x);
                        },
                        lo, hi, need, h, res, scratch, p.err);
                const uint32_t tau = lo;
                // ordered compaction: thread i owns entries [i*per, (i+1)*per)
                const uint32_t per = (m + kThreads - 1) / kThreads;
                const uint32_t j0 = min(m, tid * per), j1 = min(m, j0 + per);
                uint32_t e = 0, total;
                for (uint32_t j = j0; j < j1; ++j) e += ent[j].x == tau;
                const uint32_t ebase = block_excl_scan(e, total, scratch);
                uint32_t tie = ebase, cnt = 0;
                for (uint32_t j = j0; j < j1; ++j) {
                    const uint32_t k = ent[j].x;
                    cnt += k > tau || (k == tau && tie < need);
                    tie += k == tau;
                }
                uint32_t o = block_excl_scan(cnt, nsel, scratch);
                tie = ebase;
                for (uint32_t j = j0; j < j1; ++j) {
                    const uint2 v = ent[j];
                    if (v.x > tau || (v.x == tau && tie < need)) {
                        if (o < topk) sel[o] = static_cast<int32_t>(v.y);
                        ++o;
                    }
                    tie += v.x == tau;
                }
            } else {
                // ---- heavy ties: the same steps over the list in global memory ----
                uint32_t* E = reinterpret_cast<uint32_t*>(smem + kSelEntOff);   // per sub-segment: keys == tau
                uint32_t* G = reinterpret_cast<uint32_t*>(smem + kSelGOff);     // per sub-segment: keys selected
#pragma unroll 1
                for (int pass = 0; pass < 4 && lo != hi; ++pass)
                    radix_pass(
                        [&](auto add) {
                            for (int k = warp; k < nseg; k += kWarps) {
                                const uint2* src = glist + seg_start(p, k);
                                const uint32_t cnt = seg_cnt(k);
                                for (uint32_t j = lane; j < cnt; j += 32) add(__ldcg(src + j).x);
                            }
                        },
                        lo, hi, need, h, res, scratch, p.err);
                const uint32_t tau = lo;
                for (int k = warp; k < nseg; k += kWarps) {
                    const uint2* src = glist + seg_start(p, k);
                    const uint32_t cnt = seg_cnt(k);
                    uint32_t e = 0, g = 0;
                    for (uint32_t j = lane; j < cnt; j += 32) {
                        const uint32_t key = __ldcg(src + j).x;
                        e += key == tau;
                        g += key > tau;
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        e += __shfl_xor_sync(0xffffffffu, e, o);
                        g += __shfl_xor_sync(0xffffffffu, g, o);
                    }
                    if (lane == 0) {
                        E[k] = e;
                        G[k] = g;
                    }
                }
                __syncthreads();
                const uint32_t etotal = block_scan_array(E, nseg, scratch);   // E[k]: ties before sub-segment k
                // sub-segment k takes its keys above tau and its share of the first `need` ties
                for (int k = tid; k < nseg; k += kThreads) {
                    const uint32_t eb = E[k], ek = (k + 1 < nseg ? E[k + 1] : etotal) - eb;
                    G[k] += eb >= need ? 0u : min(ek, need - eb);
                }
                __syncthreads();
                nsel = block_scan_array(G, nseg, scratch);   // G[k]: first output slot of sub-segment k
                for (int k = warp; k < nseg; k += kWarps) {
                    const uint2* src = glist + seg_start(p, k);
                    const uint32_t cnt = seg_cnt(k);
                    uint32_t tie = E[k], o = G[k];
                    for (uint32_t j0 = 0; j0 < cnt; j0 += 32) {
                        const uint32_t j = j0 + lane;
                        const uint2 v = j < cnt ? __ldcg(src + j) : make_uint2(0u, 0u);
                        const bool eq = j < cnt && v.x == tau;
                        const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
                        const uint32_t my_tie = tie + __popc(eqb & ((1u << lane) - 1u));
                        const bool take = j < cnt && (v.x > tau || (eq && my_tie < need));
                        const uint32_t tb = __ballot_sync(0xffffffffu, take);
                        const uint32_t at = o + __popc(tb & ((1u << lane) - 1u));
                        if (take && at < topk) sel[at] = static_cast<int32_t>(v.y);
                        tie += __popc(eqb);
                        o += __popc(tb);
                    }
                }
            }
            if (tid == 0 && nsel != topk) atomicOr(p.err, ERR_TOPK_STATE);
        }
    }
    __syncthreads();
    stamp(p, 5);
    if (tid == 0) {
        __threadfence();
        red_release_add(p.ctrl + kCtrlWordReady + t, 1u);
    }
}

// Selection by position (no scoring): query t takes the last min(n_t, window)
// visible positions, ascending, then -1 padding to topk.  With window = topk and
// n_t <= topk for every query this is exactly the top-k (everything is
// selected), so the scoring phases can be skipped; with a small window it is
// sliding-window attention.
__device__ void phase_select_pos(const StepParams& p)
{
    const int64_t total = (int64_t)p.T * p.topk;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < total; i += (int64_t)gridDim.x * kThreads) {
        const int t = static_cast<int>(i / p.topk), j = static_cast<int>(i % p.topk);
        const int pos_t = query_pos_rt(p, t);
        const int cnt = min(pos_t + 1, p.window);
        p.sel[(int64_t)t * p.sel_ld + j] = j < cnt ? pos_t + 1 - cnt + j : -1;
    }
}

// ==================================================================================
// Phase 4: sparse attention, one work item per (query t, row split).  When the
// step selected the rows itself, an item starts as soon as its query's
// selection is flagged; with selection by position the rows follow from the
// query position directly.  Warp 4 gathers whole 2 KiB token rows (K then V of
// the 4 groups) by bulk async copy into a 6-stage ring of 16-row tiles; warp
// g < 4 owns KV group g, i.e. query heads 16g .. 16g+15 -- the 16 rows of an
// m16n8k16 tile, so nothing is padded.  Online softmax in the exp2 domain; the
// partial (max, sum, output) of every head goes to global memory and the item
// raises its query's done counter.
// ==================================================================================
constexpr int kAttStages = 6;
constexpr int kRowBytes = 2048;
constexpr int kPitch = 2064;                                     // bank-conflict-free ldmatrix rows
constexpr int kRowIdxOff = kAttStages * kTileRows * kPitch;      // [stage][16] row index (-1: none)
constexpr int kSelSOff = kRowIdxOff + kAttStages * kTileRows * 4;   // [kMaxRowsPerSplit] the item's rows
static_assert(kSelSOff + kMaxRowsPerSplit * 4 <= kDataBytes, "attention buffers fit");
static_assert(kBarAttEmpty + kAttStages <= kBarSlots, "attention mbarriers fit");

__device__ void phase_attend(const StepParams& p, uint8_t* smem, uint64_t* bars, bool wait_sel, int* ok_s)
{
    uint8_t* ring = smem;
    int32_t* rowidx = reinterpret_cast<int32_t*>(smem + kRowIdxOff);
    int32_t* sel_s = reinterpret_cast<int32_t*>(smem + kSelSOff);
    uint64_t* full = bars + kBarAttFull;
    uint64_t* empty = bars + kBarAttEmpty;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, c = lane & 3;
    constexpr int kConsumers = 4, kProducer = 4;
    const float sm_scale = kLog2e * rsqrtf(static_cast<float>(kD));
    const bool by_pos = (p.phases & kPhaseSelectPos) != 0;

    int phase_base = 0;   // tiles consumed by this block so far (mbarrier phase bookkeeping)
    if (tid == 0) {
        for (int s = 0; s < kAttStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumers);
        }
        fence_mbar_init();
    }
    __syncthreads();

    for (int r = 0;; ++r) {
        const int i = item_of(r);
        if (i >= p.T * p.nsplit) break;
        const int t = i / p.nsplit, split = i % p.nsplit;
        const int pos_t = query_pos_rt(p, t);
        bool sel_ok = true;
        if (wait_sel) {   // the query's selection is written (phase 3 flags it)
            if (tid == 0) *ok_s = wait_counter(p, p.ctrl + kCtrlWordReady + t, 1u) ? 1 : 0;
            __syncthreads();
            sel_ok = *ok_s != 0;
        }
        if (r == 0) stamp(p, 6);
        const int rows_t = min(p.rows, pos_t + 1);
        const int r0 = split * p.rows_per_split;
        const int r1 = sel_ok ? min(r0 + p.rows_per_split, rows_t) : r0;   // no selection: an empty partial
        const int ntile = r1 > r0 ? (r1 - r0 + kTileRows - 1) / kTileRows : 0;

        bool failed = false;
        float oacc[16][4];
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) oacc[k][0] = oacc[k][1] = oacc[k][2] = oacc[k][3] = 0.f;

        if (warp == kProducer) {
            // producer: the item's rows, validated, then gathered whole
            if (by_pos) {
                const int cnt = min(pos_t + 1, p.window);   // row j of the window: pos_t + 1 - cnt + j
                for (int j = lane; j < r1 - r0; j += 32) sel_s[j] = pos_t + 1 - cnt + r0 + j;
            } else {
                const int32_t* selrow = p.sel + (int64_t)t * p.sel_ld + r0;
                int32_t v[kMaxRowsPerSplit / 32];   // every load in flight before the first store
#pragma unroll
                for (int u = 0; u < kMaxRowsPerSplit / 32; ++u) {
                    const int j = lane + u * 32;
                    v[u] = j < r1 - r0 ? __ldcg(selrow + j) : -1;
                }
#pragma unroll
                for (int u = 0; u < kMaxRowsPerSplit / 32; ++u)
                    if (lane + u * 32 < r1 - r0) sel_s[lane + u * 32] = v[u];
            }
            __syncwarp();
            for (int k = 0; k < ntile; ++k) {
                const int kk = phase_base + k;
                const int stage = kk % kAttStages;
                if (kk >= kAttStages && !mbar_wait(&empty[stage], ((kk / kAttStages) - 1) & 1, p.err)) {
                    failed = true;
                    break;
                }
                uint8_t* dst = ring + stage * kTileRows * kPitch;
                int s = -1;
                bool valid = false;
                if (lane < kTileRows) {
                    const int j = k * kTileRows + lane;
                    if (r0 + j < r1) {
                        s = sel_s[j];
                        valid = s >= 0 && s <= pos_t && s < p.L;
                        if (s >= 0 && !valid) atomicOr(p.err, ERR_BAD_INDEX);
                    }
                    rowidx[stage * kTileRows + lane] = valid ? s : -1;
                }
                const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
                // Rows with nothing to load get a zero V half, so P = 0 never meets stale data.
                uint32_t none = ~vmask & 0xFFFFu;
                while (none) {
                    const int z = __ffs(none) - 1;
                    none &= none - 1;
                    uint4* v = reinterpret_cast<uint4*>(dst + z * kPitch + kRowBytes / 2);
                    v[lane] = make_uint4(0u, 0u, 0u, 0u);
                    v[lane + 32] = make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_expect_tx(&full[stage], __popc(vmask) * kRowBytes);
                __syncwarp();
                if (valid) bulk_g2s(dst + lane * kPitch, p.kv + (int64_t)s * p.kv_ld, kRowBytes, &full[stage]);
            }
        } else if (warp < kConsumers) {
            const int grp = warp;
            uint32_t qa[8][4];
            const uint16_t* qbp = p.q + ((int64_t)t * kH + grp * 16) * kD;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                qa[kk][0] = __ldg(reinterpret_cast<const uint32_t*>(qbp + gq * kD + kk * 16 + 2 * c));
                qa[kk][1] = __ldg(reinterpret_cast<const uint32_t*>(qbp + (gq + 8) * kD + kk * 16 + 2 * c));
                qa[kk][2] = __ldg(reinterpret_cast<const uint32_t*>(qbp + gq * kD + kk * 16 + 8 + 2 * c));
                qa[kk][3] = __ldg(reinterpret_cast<const uint32_t*>(qbp + (gq + 8) * kD + kk * 16 + 8 + 2 * c));
            }
            for (int k = 0; k < ntile; ++k) {
                const int kk0 = phase_base + k;
                const int stage = kk0 % kAttStages;
                if (!mbar_wait(&full[stage], (kk0 / kAttStages) & 1, p.err)) {
                    failed = true;
                    break;
                }
                const uint32_t base = smem_u32(ring + stage * kTileRows * kPitch);
                const int32_t* ridx = rowidx + stage * kTileRows;
                float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                float sodd[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int kk2 = 0; kk2 < 4; ++kk2) {
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const int key = nt * 8 + (lane & 7);
                        const int dim = kk2 * 32 + (lane >> 3) * 8;
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(base + key * kPitch + grp * 256 + dim * 2, b0, b1, b2, b3);
                        mma_bf16_16816(sacc[nt], qa[2 * kk2], b0, b1);
                        mma_bf16_16816(sodd[nt], qa[2 * kk2 + 1], b2, b3);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = nt * 8 + 2 * c + (e & 1);
                        const float z = sacc[nt][e] + sodd[nt][e];
                        sacc[nt][e] = ridx[key] >= 0 ? z * sm_scale : -INFINITY;
                    }
                float mx0 = fmaxf(fmaxf(sacc[0][0], sacc[0][1]), fmaxf(sacc[1][0], sacc[1][1]));
                float mx1 = fmaxf(fmaxf(sacc[0][2], sacc[0][3]), fmaxf(sacc[1][2], sacc[1][3]));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
                const float z0 = n0 == -INFINITY ? 0.f : n0, z1 = n1 == -INFINITY ? 0.f : n1;
                const float alpha0 = exp2f(m0 - z0), alpha1 = exp2f(m1 - z1);
                m0 = n0;
                m1 = n1;
                float pr[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    pr[nt][0] = exp2f(sacc[nt][0] - z0);
                    pr[nt][1] = exp2f(sacc[nt][1] - z0);
                    pr[nt][2] = exp2f(sacc[nt][2] - z1);
                    pr[nt][3] = exp2f(sacc[nt][3] - z1);
                }
                l0 = l0 * alpha0 + (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
                l1 = l1 * alpha1 + (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    oacc[e][0] *= alpha0;
                    oacc[e][1] *= alpha0;
                    oacc[e][2] *= alpha1;
                    oacc[e][3] *= alpha1;
                }
                uint32_t pa[4];
                pa[0] = pack_bf16(pr[0][0], pr[0][1]);
                pa[1] = pack_bf16(pr[0][2], pr[0][3]);
                pa[2] = pack_bf16(pr[1][0], pr[1][1]);
                pa[3] = pack_bf16(pr[1][2], pr[1][3]);
#pragma unroll
                for (int nd2 = 0; nd2 < 8; ++nd2) {
                    const int key = (lane & 7) + 8 * ((lane >> 3) & 1);
                    const int dim = nd2 * 16 + 8 * (lane >> 4);
                    uint32_t v0, v1, v2, v3;
                    ldsm_x4_t(base + key * kPitch + kRowBytes / 2 + grp * 256 + dim * 2, v0, v1, v2, v3);
                    mma_bf16_16816(oacc[2 * nd2], pa, v0, v1);
                    mma_bf16_16816(oacc[2 * nd2 + 1], pa, v2, v3);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
            }
        }
        if (__syncthreads_or(failed)) {
            // A bounded wait ran out: let the copies in flight land; the partial is empty.
            if (tid == kProducer * 32)
                for (int k = max(0, ntile - kAttStages); k < ntile; ++k)
                    mbar_wait(&full[(phase_base + k) % kAttStages], ((phase_base + k) / kAttStages) & 1, p.err);
            __syncthreads();
            m0 = m1 = -INFINITY;
            l0 = l1 = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k) oacc[k][0] = oacc[k][1] = oacc[k][2] = oacc[k][3] = 0.f;
        }
        if (warp < kConsumers) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
            l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
            const int h0 = warp * 16 + gq, h1 = h0 + 8;
            const int64_t part = (int64_t)t * p.nsplit + split;
            if (c == 0) {
                p.pml[part * kH + h0] = make_float2(m0, l0);
                p.pml[part * kH + h1] = make_float2(m1, l1);
            }
            float* o0 = p.po + (part * kH + h0) * kD;
            float* o1 = p.po + (part * kH + h1) * kD;
#pragma unroll
            for (int nd = 0; nd < 16; ++nd) {
                *reinterpret_cast<float2*>(o0 + nd * 8 + 2 * c) = make_float2(oacc[nd][0], oacc[nd][1]);
                *reinterpret_cast<float2*>(o1 + nd * 8 + 2 * c) = make_float2(oacc[nd][2], oacc[nd][3]);
            }
        }
        phase_base += ntile;
        __syncthreads();
        if (tid == 0) red_release_add(p.ctrl + kCtrlWordDone + t, 1u);   // this split of query t is written
    }
}

// ==================================================================================
// Phase 5: merge the splits of each (query, head) in split order, one warp per
// item (query t, head h, half of the 128 dims), starting once every split of
// its query is done (its counter; no grid barrier).  Lane s loads split s's
// (max, sum); every lane loads all splits' outputs for its two dims, all loads
// in flight at once; the max, the weights and the denominator come by warp
// shuffles, the sink joins the denominator with no value row.
// ==================================================================================
__device__ void phase_merge(const StepParams& p, int* ok_s)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int P = 2;                          // halves of the 128 dims per (t, h); two dims per lane
    static_assert((kH * P) % kWarps == 0, "a block's items of one round belong to one query");
    const int items = p.T * kH * P;
    const int ns = p.nsplit;                      // <= kMaxSplitsQ
    for (int i0 = blockIdx.x * kWarps; i0 < items; i0 += gridDim.x * kWarps) {
        // One thread waits for the query's splits, then the whole block goes on: the
        // waiting stays out of the warps' loads.
        const int t = i0 / (kH * P);
        if (threadIdx.x == 0) *ok_s = wait_counter(p, p.ctrl + kCtrlWordDone + t, static_cast<uint32_t>(ns)) ? 1 : 0;
        __syncthreads();
        const bool ok = *ok_s != 0;
        __syncthreads();   // every thread has read the flag before the next round writes it
        const int i = i0 + warp;
        if (!ok || i >= items) continue;
        const int h = (i / P) % kH, part = i % P;
        const float2* ml = p.pml + (int64_t)t * ns * kH + h;
        const int d0 = part * (kD / P) + lane * 2;
        const float* po = p.po + ((int64_t)t * ns * kH + h) * kD + d0;
        const float2 mine = lane < ns ? __ldcg(ml + (int64_t)lane * kH) : make_float2(-INFINITY, 0.f);
        float2 o[kMaxSplitsQ];
#pragma unroll
        for (int s = 0; s < kMaxSplitsQ; ++s)
            o[s] = s < ns ? __ldcg(reinterpret_cast<const float2*>(po + (int64_t)s * kH * kD)) : make_float2(0.f, 0.f);
        const float sink = p.sink != nullptr ? p.sink[h] * kLog2e : -INFINITY;
        float M = fmaxf(mine.x, sink);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float wmine = mine.x == -INFINITY ? 0.f : exp2f(mine.x - M);
        float den = wmine * mine.y;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int s = 0; s < kMaxSplitsQ; ++s) {   // splits in order
            const float w = __shfl_sync(0xffffffffu, wmine, s);
            if (s < ns) {
                x0 = fmaf(w, o[s].x, x0);
                x1 = fmaf(w, o[s].y, x1);
            }
        }
        const float dd = den + ((p.sink != nullptr && M != -INFINITY) ? exp2f(sink - M) : 0.f);
        const float inv = dd > 0.f ? 1.0f / dd : 0.f;
        *reinterpret_cast<uint32_t*>(p.out + ((int64_t)t * kH + h) * kD + d0) = pack_bf16(x0 * inv, x1 * inv);
    }
}

// ==================================================================================
// Launch view: the histogram buffer of this launch's epoch (when the launch
// counts one), and the query positions when they come from device memory (so
// that one CUDA graph of the step serves every decode position; a position
// outside [0, L) is clamped and flagged).  Returns the epoch (thread 0).
__device__ uint32_t init_launch_view(const StepParams& p, bool counts)
{
    uint32_t e = 0u;
    if (threadIdx.x == 0) {
        e = p.ctrl != nullptr ? *reinterpret_cast<volatile uint32_t*>(p.ctrl + kCtrlWordEpoch) : 0u;
        g_view.hist = counts && p.ctrl != nullptr ? p.ctrl + kCtrlBytes / 4 + (e & 1u) * kHistWords : nullptr;
    }
    if (p.pos_dev != nullptr && threadIdx.x < 32) {
        int v = 0;
        if (threadIdx.x < p.T) {
            v = __ldcg(p.pos_dev + threadIdx.x);
            if (v < 0 || v >= p.L) {
                if (blockIdx.x == 0) atomicOr(p.err, ERR_BAD_POS);
                v = min(max(v, 0), p.L - 1);
            }
        }
        if (threadIdx.x < kMaxT) g_view.pos[threadIdx.x] = v;
        int n = threadIdx.x < p.T ? v + 1 : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) n = max(n, __shfl_xor_sync(0xffffffffu, n, o));
        if (threadIdx.x == 0) g_view.n_max = n;
    }
    return e;
}

// The indexer stage as a kernel of its own: one block per SM, 17 warps.  With a
// workspace it also counts the first radix pass into the launch's histogram.
template <bool FP8>
__global__ void __launch_bounds__(kIdxThreads, 1) index_kernel(const __grid_constant__ CUtensorMap kmap, const StepParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOffset);
    __shared__ uint32_t tmem_slot;
    // the cooperative kernel that consumes the scores may be launched now: its
    // blocks take the SMs this grid leaves and wait for its completion
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    init_launch_view(p, p.hist_bound != 0);
    if (p.hist_bound && p.ctrl != nullptr && blockIdx.x == 0 && threadIdx.x == 0) check_ctrl_words(p);
    __syncthreads();
    stamp(p, 0);
    if (p.trace != nullptr && threadIdx.x == 0) p.trace[(int64_t)blockIdx.x * kTraceSlots + 28] = clock64();
    phase_index<FP8>(kmap, p, smem, bars, &tmem_slot);
    __syncthreads();
    stamp(p, 1);
}

// Stages 2 and 3 (and the first radix pass of caller-provided scores): one
// cooperative launch, one block per SM.
__global__ void __launch_bounds__(kThreads, 1) step_kernel(const StepParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOffset);
    __shared__ __align__(16) uint32_t scratch[64];
    __shared__ uint32_t res[3];
    __shared__ int ok_s;
    __shared__ uint32_t epoch_s;

    const uint32_t e = init_launch_view(p, (p.phases & kPhaseTopk) && (p.hist_bound || (p.phases & kPhaseHistScores)));
    if (threadIdx.x == 0) epoch_s = e;
    __syncthreads();
    // The other histogram buffer starts the next launch at zero.
    if (p.ctrl != nullptr) {
        uint32_t* next = p.ctrl + kCtrlBytes / 4 + ((epoch_s + 1u) & 1u) * kHistWords;
        for (int i = blockIdx.x * kThreads + threadIdx.x; i < kHistWords; i += gridDim.x * kThreads) next[i] = 0u;
    }

    GridBarrier gb{p.ctrl, gridDim.x};
    // Stamps (when tracing): 0 start and 1 first stage done (the indexer kernel's
    // when it ran), 2 extraction start (after the barrier), 3 extraction done, 4/5
    // selection (blocks < T), 6 first attention item starts, 7 this block's
    // attention items done, 9 its merge items done, 30 end, 31 this kernel's
    // start; SM clock: 28 first kernel's start, 27 this kernel's start, 29 end.
    bool ok = true;
    const bool checked = p.hist_bound != 0;   // the indexer kernel checked the control words
    if (p.ctrl != nullptr && !checked) gb.enter();
    // Launched as a programmatic dependent of the indexer kernel: everything above
    // touches nothing that grid writes; its scores and histogram are read below.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (p.trace != nullptr && threadIdx.x == 0) {   // this kernel's own start: SM clock and time
        p.trace[(int64_t)blockIdx.x * kTraceSlots + 27] = clock64();
        stamp(p, 31);
    }
    const bool own_first = !p.hist_bound;   // no indexer kernel ran before this one
    if (own_first) {
        stamp(p, 0);
        if (p.trace != nullptr && threadIdx.x == 0) p.trace[(int64_t)blockIdx.x * kTraceSlots + 28] = clock64();
    }
    if (p.phases & kPhaseHistScores) phase_hist_scores(p, smem);
    if (own_first) stamp(p, 1);
    if (p.phases & kPhaseTopk) {
        if (!checked) {
            ok = gb.sync(p, &ok_s);
        } else if (p.ctrl != nullptr) {
            // Nothing before the extraction depends on another block of this grid:
            // the scores, histogram and group maxima are complete once the indexer
            // kernel is, so no grid barrier; only its verdict on the control words.
            if (threadIdx.x == 0) ok_s = *reinterpret_cast<volatile uint32_t*>(p.ctrl + kCtrlWordBad) == 0u;
            __syncthreads();
            ok = ok_s != 0;
        }
        stamp(p, 2);
        if (ok) phase_extract(p, smem, bars, res, scratch);
        stamp(p, 3);
        if (ok) {
            phase_select(p, smem, res, scratch, &ok_s);
        } else if (blockIdx.x < p.T && threadIdx.x == 0) {
            red_release_add(p.ctrl + kCtrlWordReady + blockIdx.x, 1u);   // nothing to wait for downstream
        }
    }
    if (p.phases & kPhaseSelectPos) phase_select_pos(p);   // the attention derives the same rows itself
    if (p.phases & kPhaseAttend) {
        if (ok) phase_attend(p, smem, bars, (p.phases & kPhaseTopk) != 0, &ok_s);
        stamp(p, 7);
        if (ok) phase_merge(p, &ok_s);
        __syncthreads();
        stamp(p, 9);
    }
    if (p.ctrl != nullptr) barrier_exit(p);
    if (p.trace != nullptr && threadIdx.x == 0) {
        p.trace[(int64_t)blockIdx.x * kTraceSlots + 29] = clock64();
        stamp(p, 30);
    }
}

bool g_configured[64][3] = {};
bool g_no_pdl[64] = {};

}  // namespace

int step_smem_bytes() { return kStepSmem; }

cudaError_t launch_step(const CUtensorMap* kmap, const StepParams& p, bool fp8, cudaStream_t s, cudaEvent_t mid_event)
{
    int dev = 0;
    cudaGetDevice(&dev);
    const bool cache = dev >= 0 && dev < 64;
    if (p.phases & kPhaseIndex) {
        auto kern = fp8 ? index_kernel<true> : index_kernel<false>;
        if (!cache || !g_configured[dev][fp8]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kStepSmem);
            if (e != cudaSuccess) return e;
            if (cache) g_configured[dev][fp8] = true;
        }
        StepParams q = p;
        q.hist_bound = (p.phases & kPhaseTopk) != 0 ? 1 : 0;
        kern<<<p.grid, kIdxThreads, kStepSmem, s>>>(*kmap, q);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        if (mid_event != nullptr && (e = cudaEventRecord(mid_event, s)) != cudaSuccess) return e;
    }
    StepParams q = p;
    q.phases &= ~kPhaseIndex;
    q.hist_bound = (p.phases & kPhaseIndex) != 0 && (p.phases & kPhaseTopk) != 0 ? 1 : 0;
    if (q.phases == 0) return cudaSuccess;
    if (!cache || !g_configured[dev][2]) {
        cudaError_t e = cudaFuncSetAttribute(step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStepSmem);
        if (e != cudaSuccess) return e;
        if (cache) g_configured[dev][2] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kStepSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    // after the indexer kernel: a programmatic dependent launch (its launch overlaps
    // the indexer's tail), unless the device turned that down once
    const bool pdl = (p.phases & kPhaseIndex) != 0 && !(cache && g_no_pdl[dev]);
    cfg.numAttrs = pdl ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, step_kernel, q);
    if (e != cudaSuccess && pdl) {
        cudaGetLastError();
        if (cache) g_no_pdl[dev] = true;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, step_kernel, q);
    }
    return e;
}

int step_max_blocks(bool fp8)
{
    (void)fp8;
    int dev = 0, sms = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaFuncSetAttribute(step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStepSmem);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, step_kernel, kThreads, kStepSmem) != cudaSuccess || n < 1)
        n = 1;
    cudaGetLastError();
    return sms * (n > 1 ? 1 : n);   // one block per SM
}

}  // namespace dsa
