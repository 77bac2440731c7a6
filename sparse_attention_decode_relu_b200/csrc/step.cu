// step.cu -- the DSA decode/verify step as one cooperative persistent kernel.
//
// NaiveAI research page (naive.ai/en/research), "NaiveRT > A DSA layer: from 29
// kernels to one": a DSA layer runs as a single cooperative kernel across 148
// CTAs in one grid.  Here one block per SM runs every phase of the step, with a
// bounded grid barrier between phases, so no kernel boundary (launch latency,
// ramp, drain) separates the stages:
//
//   1 index   : ReLU indexer scan over the key cache: TMA key tiles,
//               tcgen05.mma with fp32 accumulators in TMEM, fp32 scores plus
//               each block's per-query key range
//   2 hist    : first radix pass of the top-k, per (query, chunk) work item:
//               4096 bins over the query's key range, summed in global memory
//   3 extract : the bin holding the topk-th key; every key at or above that bin
//               goes to the query's candidate list, keys above it are counted
//               per chunk
//   4 emit    : each chunk block finds tau and the tie cut among the keys inside
//               the bin and writes its selected positions in order
//   (or)      : selection by position: the last W visible positions (the
//               short-context bypass with W = topk, sliding-window decode)
//   5 attend  : gathered sparse attention per (query, row split): whole K/V rows
//               by bulk async copy, tensor-core QK and PV, online softmax;
//               partial (max, sum, output) states to global memory
//   6 merge   : per (query, head), the splits merged in a fixed order
//
// Stage entry points run a sub-range of the phases.  Every reduction is either
// integer or in a fixed order, so results are bitwise reproducible.
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;

// ---- shared memory map (dynamic, 1024-aligned base) --------------------------
constexpr int kIdxStages = 6;
constexpr int kAttStages = 6;
constexpr int kTileRows = 16;
constexpr int kRowBytes = 2048;
constexpr int kPitch = 2064;              // bank-conflict-free ldmatrix rows
constexpr int kDataBytes = kAttStages * kTileRows * kPitch + kAttStages * kTileRows * 4 + kMaxRowsPerSplit * 4;
constexpr int kBarOffset = (kDataBytes + 127) / 128 * 128;
constexpr int kBarSlots = 64;             // mbarriers (8 bytes each) after the data region
constexpr int kStepSmem = 1024 + kBarOffset + kBarSlots * 8;


__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier among the co-resident blocks of a cooperative launch.  The
// arrival counter only grows during a launch (it is zero at launch): barrier k
// ends when it reaches k * gridDim.x.  Each block adds 1 with release semantics
// and polls with acquire loads, giving up (error bit, false) after
// kWaitLimitCycles.  The launch leaves the counter at zero again (see
// GridBarrier::enter / barrier_exit), so consecutive launches need no reset node.
// Control words: the arrival count at word 0, the exit count on the next
// 128-byte line.
constexpr int kExitWord = 32;

struct GridBarrier {
    uint32_t* count;
    uint32_t* err;
    uint32_t next;     // count value that ends the next barrier
    long long limit;   // SM clocks a wait spins before it gives up
    uint32_t extra;    // arrivals waited for beyond the grid's own (0 except under the fault hook)
    uint32_t c0 = 0, x0 = 0;   // (thread 0) both words as this block first saw them
    bool bad = false;          // (thread 0) they were not zero at launch

    // Thread 0 reads the control words at kernel entry; they are checked at the
    // first barrier, so the loads overlap the first phase.
    __device__ void enter()
    {
        if (threadIdx.x == 0) {
            c0 = *reinterpret_cast<volatile uint32_t*>(count);
            x0 = *reinterpret_cast<volatile uint32_t*>(count + kExitWord);
        }
    }

    __device__ bool sync(int* ok_s)
    {
        __syncthreads();
        if (threadIdx.x == 0) {
            // Before its first arrival a block can see at most gridDim.x - 1
            // arrivals and no exit (nobody passes the first barrier without it);
            // anything else means the words were not zero at launch.  Such a
            // block flags it and takes no part in the barriers.
            if (next == gridDim.x && (x0 != 0u || c0 >= gridDim.x)) {
                bad = true;
                atomicOr(err, ERR_WORKSPACE_STATE);
            }
            bool ok = !bad;
            if (ok) {
                const uint32_t target = next + extra;
                asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(count) : "memory");
                const long long t0 = clock64();
                while (ld_acquire(count) < target) {
                    if (clock64() - t0 > limit) {
                        atomicOr(err, ERR_WAIT_TIMEOUT);
                        ok = false;
                        break;
                    }
                }
            }
            *ok_s = ok ? 1 : 0;
        }
        __syncthreads();
        next += gridDim.x;
        return *ok_s != 0;
    }
};

__device__ __forceinline__ void barrier_exit(const StepParams& p)
{
    if (threadIdx.x == 0) {
        uint32_t old;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                     : "=r"(old)
                     : "l"(p.bar_ctrl + kExitWord)
                     : "memory");
        if (old == gridDim.x - 1u) {
            p.bar_ctrl[0] = 0u;
            p.bar_ctrl[kExitWord] = 0u;
        }
    }
}

// The query positions of this launch (from the launch parameters, or read from
// device memory at launch) and the furthest visible position + 1.
struct PosView {
    int32_t pos[kMaxT];
    int32_t n_max;
};
__shared__ PosView g_qpos;

// Position of query k: the launch parameter (constant bank), or the view filled
// from device memory at launch.
__device__ __forceinline__ int query_pos(const StepParams& p, int k)
{
    return p.pos_dev != nullptr ? g_qpos.pos[k] : p.pos[k];
}
__device__ __forceinline__ int visible_max(const StepParams& p)
{
    return p.pos_dev != nullptr ? g_qpos.n_max : p.n_max;
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
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t& total, uint32_t* scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t x = warp_incl_scan(v);
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const uint32_t w = lane < kWarps ? scratch[lane] : 0u;
        const uint32_t wi = warp_incl_scan(w);
        if (lane < kWarps) scratch[lane] = wi;
    }
    __syncthreads();
    const uint32_t before = warp ? scratch[warp - 1] : 0u;
    total = scratch[kWarps - 1];
    __syncthreads();
    return before + x - v;
}

// Sum over the block in a fixed order (warp tree, then warps 0..7); the
// barriers also order the shared-memory writes made before the call.
__device__ __forceinline__ float block_sum_f(float v, uint32_t* scratch)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = __float_as_uint(v);
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += __uint_as_float(scratch[w]);
    __syncthreads();
    return s;
}

__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* scratch)
{
    uint32_t total;
    block_excl_scan(v, total, scratch);
    return total;
}

__device__ __forceinline__ void block_minmax(uint32_t& lo, uint32_t& hi, uint32_t* scratch)
{
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
    for (int w = 1; w < kWarps; ++w) {
        lo = min(lo, scratch[w]);
        hi = max(hi, scratch[32 + w]);
    }
    __syncthreads();
}

// Append the values x of the lanes with `take` set to v[*count ..] (one shared
// atomic per warp; entries past cap are counted but not stored).  Every lane of
// the warp must call it.
template <typename V>
__device__ __forceinline__ void warp_append(bool take, V x, V* v, uint32_t* count, uint32_t cap)
{
    const int lane = threadIdx.x & 31;
    const uint32_t bal = __ballot_sync(0xffffffffu, take);
    if (!bal) return;
    uint32_t base = 0;
    if (lane == 0) base = atomicAdd(count, static_cast<uint32_t>(__popc(bal)));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (take) {
        const uint32_t at = base + __popc(bal & ((1u << lane) - 1u));
        if (at < cap) v[at] = x;
    }
}

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

// Bin b of an NB-bin histogram in shared memory holding the need-th largest
// entry: #(bins > b) < need <= #(bins >= b).  res = {b, #(bins > b), found}.
template <int NB>
__device__ void find_from_top(const uint32_t* h, uint32_t need, uint32_t* res, uint32_t* scratch)
{
    constexpr int PER = NB / kThreads;
    const int top = NB - PER * threadIdx.x;   // thread 0 owns the highest bins
    uint32_t cnt[PER];
    uint32_t sum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        cnt[i] = h[top - 1 - i];
        sum += cnt[i];
    }
    if (threadIdx.x == 0) res[2] = 0;
    uint32_t total;
    uint32_t run = block_excl_scan(sum, total, scratch);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        if (run < need && run + cnt[i] >= need) {
            res[0] = static_cast<uint32_t>(top - 1 - i);
            res[1] = run;
            res[2] = 1;
        }
        run += cnt[i];
    }
    __syncthreads();
}

// Work item i of `items` assigned to this block in round r (i = block + r*grid).
__device__ __forceinline__ int item_of(int r) { return blockIdx.x + r * gridDim.x; }

// ==================================================================================
// Phase 1: indexer scan on the fifth-generation tensor cores.  A tile of 128 keys
// is the M side of tcgen05.mma (kind::f16: bf16 operands, fp32 accumulators in
// tensor memory), the T x 16 indexer query heads the N side, the 64 dims K (four
// K = 16 steps).  TMA brings key tiles into a ring; E4M3 tiles are widened to
// bf16 (exactly) into a 128B-swizzled buffer.  One thread issues the MMAs; the
// accumulators of consecutive tiles alternate between two TMEM buffers so that
// the epilogue of one tile overlaps the MMA of the next.  Epilogue: each thread
// owns one key row (a TMEM lane) and, per query, applies ReLU, the head weights,
// a fixed-order sum over the 16 heads and the per-token scale.
// ==================================================================================
constexpr uint32_t kTmemCols = 256;        // two accumulator buffers of 128 columns
constexpr int kMmaBar = 40;                // the two MMA-completion mbarriers
constexpr int kTileBytesBf16 = kKeyTile * kDI * 2;   // 16 KiB, one 128 x 64 bf16 operand tile
static_assert(kIdxStages * kTileBytesBf16 + 2 * kTileBytesBf16 + kTileBytesBf16 + kMaxT * kHI * 4 +
                  (kIdxStages + 4) * kKeyTile * 4 <= kDataBytes, "indexer buffers fit the data region");
static_assert(kMmaBar + 6 <= kBarSlots && kIdxStages + 1 <= 8, "indexer mbarriers fit");

template <bool FP8>
__device__ void phase_index(const CUtensorMap& kmap, const CUtensorMap& smap, const StepParams& p, uint8_t* smem,
                            uint64_t* bars, uint32_t* scratch, uint32_t* tmem_slot)
{
    constexpr int raw_bytes = kKeyTile * kDI * (FP8 ? 1 : 2);
    uint8_t* ring = smem;                                                  // [kIdxStages][raw_bytes]
    uint8_t* cvt = ring + kIdxStages * raw_bytes;                          // FP8: [2][16 KiB] bf16 tiles
    uint8_t* qsw = cvt + (FP8 ? 2 * kTileBytesBf16 : 0);                   // [128 rows][128 B] queries
    float* w_s = reinterpret_cast<float*>(qsw + kTileBytesBf16);           // [8][16]
    float* sc_s = w_s + kMaxT * kHI;                                       // [kIdxStages][128] scales
    float* scl = sc_s + kIdxStages * kKeyTile;                             // [2 halves][2][128] tile scales
    uint64_t* full = bars;                  // [kIdxStages] key tile landed
    uint64_t* setup = bars + kIdxStages;
    uint64_t* mmab = bars + kMmaBar;        // [2] MMAs of the tile in TMEM buffer b complete
    uint64_t* convb = mmab + 2;             // [2] every thread is done with the raw tile of buffer b
    uint64_t* tfree = mmab + 4;             // [2] every thread is done reading TMEM buffer b

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = p.T;
    const int ntiles = (visible_max(p) + kKeyTile - 1) / kKeyTile;
    const bool scaled = p.scale != nullptr;
    const uint32_t tile_tx = raw_bytes + (scaled ? kKeyTile * 4 : 0);
    auto tile_of = [&](int it) { return blockIdx.x + it * static_cast<int>(gridDim.x); };
    auto load_tile = [&](int stage, int tile) {
        mbar_arrive_expect_tx(&full[stage], tile_tx);
        tma_load_2d(ring + stage * raw_bytes, &kmap, 0, tile * kKeyTile, &full[stage]);
        if (scaled) tma_load_1d(sc_s + stage * kKeyTile, &smap, tile * kKeyTile, &full[stage]);
    };

    int issued = 0;   // key tiles requested by thread 0
    if (tid == 0) {
        prefetch_tmap(&kmap);
        if (scaled) prefetch_tmap(&smap);
        for (int s = 0; s <= kIdxStages; ++s) mbar_init(&bars[s], 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&mmab[b], 1);
            mbar_init(&convb[b], kThreads);
            mbar_init(&tfree[b], kThreads);
        }
        fence_mbar_init();
        mbar_arrive_expect_tx(setup, T * kHI * 4);
        bulk_g2s(w_s, p.w, T * kHI * 4, setup);
        for (int s = 0; s < kIdxStages && tile_of(s) < ntiles; ++s) {
            load_tile(s, tile_of(s));
            ++issued;
        }
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    // The indexer queries as the B operand: row r = t*16 + j, 16-byte chunk c at
    // r*128 + (c ^ (r & 7))*16 (the 128B swizzle); rows >= T*16 are never read.
    {
        uint4 v[kMaxT * kHI * 8 / kThreads];   // every load in flight before the first store
#pragma unroll
        for (int u = 0; u < kMaxT * kHI * 8 / kThreads; ++u) {
            const int i = tid + u * kThreads;
            v[u] = i < T * kHI * 8 ? __ldg(reinterpret_cast<const uint4*>(p.q_idx) + i) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kMaxT * kHI * 8 / kThreads; ++u) {
            const int i = tid + u * kThreads, r = i >> 3, c = i & 7;
            if (i < T * kHI * 8) *reinterpret_cast<uint4*>(qsw + r * 128 + ((c ^ (r & 7)) << 4)) = v[u];
        }
    }
    // Counters the top-k phases accumulate into start at zero.
    for (int i = blockIdx.x * kThreads + tid; i < p.zero_words; i += gridDim.x * kThreads) p.zero[i] = 0u;
    fence_proxy_async_smem();   // the queries are read by the tensor cores (async proxy)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = mbar_wait(setup, 0, p.err);

    // Warp w reads TMEM lanes 32*(w%4) .. +31 (its key rows) and the columns of
    // queries [qa, qb): warps 0-3 the first ceil(T/2) queries, warps 4-7 the rest.
    const int quad = warp & 3, half = warp >> 2;
    const int tsplit = (T + 1) >> 1;
    const int qa = half ? tsplit : 0, qb = half ? T : tsplit;
    const int row = quad * 32 + lane;
    int pos_q[4];
    uint32_t klo[4], khi[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        pos_q[u] = -1;
#pragma unroll
        for (int i = 0; i < kMaxT; ++i)
            if (i == qa + u) pos_q[u] = query_pos(p, i);
        klo[u] = 0xFFFFFFFFu;
        khi[u] = 0u;
    }
    const uint32_t idesc = umma_idesc_bf16(kKeyTile, T * kHI);
    const uint64_t bdesc = umma_desc_sw128(smem_u32(qsw));

    int mma_issued = 0, mma_done = 0;   // (thread 0) tiles whose MMAs were issued / waited for
    float* my_scl = scl + half * 2 * kKeyTile;   // this half's copy: written and read by the same thread
    // Epilogue of local tile e: wait for its MMAs, then scores from TMEM buffer e & 1.
    auto epilogue = [&](int e) -> bool {
        const int b = e & 1;
        if (!mbar_wait(&mmab[b], (e >> 1) & 1, p.err)) return false;
        tc_fence_after();
        if (qa < qb) {
            const int s = tile_of(e) * kKeyTile + row;
            const float scale = my_scl[b * kKeyTile + row];
            const uint32_t tbase = tmem + static_cast<uint32_t>((quad * 32) << 16) + b * 128 + qa * kHI;
            // Up to four queries: two TMEM loads in flight, one wait; the 16-head sum as
            // four interleaved partial sums over heads {j, j+4, j+8, j+12}, combined in
            // a fixed order.
            uint32_t r[2][32];
            tmem_ld32_nowait(tbase, r[0]);
            if (qb - qa > 2) tmem_ld32_nowait(tbase + 2 * kHI, r[1]);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int t = qa + u;
                if (t < qb) {
                    const float4* w4 = reinterpret_cast<const float4*>(w_s + t * kHI);
                    const float* v = reinterpret_cast<const float*>(&r[u >> 1][(u & 1) * 16]);
                    float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int g4 = 0; g4 < 4; ++g4) {
                        const float4 w = w4[g4];
                        part[0] = fmaf(fmaxf(v[g4 * 4 + 0], 0.f), w.x, part[0]);
                        part[1] = fmaf(fmaxf(v[g4 * 4 + 1], 0.f), w.y, part[1]);
                        part[2] = fmaf(fmaxf(v[g4 * 4 + 2], 0.f), w.z, part[2]);
                        part[3] = fmaf(fmaxf(v[g4 * 4 + 3], 0.f), w.w, part[3]);
                    }
                    const float acc = ((part[0] + part[1]) + (part[2] + part[3])) * scale;
                    if (s < p.L) {
                        if (s <= pos_q[u]) {
                            p.scores[(int64_t)t * p.ld + s] = acc;
                            const uint32_t k = score_key(acc);
                            klo[u] = min(klo[u], k);
                            khi[u] = max(khi[u], k);
                        } else {
                            p.scores[(int64_t)t * p.ld + s] = -INFINITY;
                        }
                    }
                }
            }
        }
        tc_fence_before();
        mbar_arrive(&tfree[b]);
        return true;
    };

    // Steady state without block-wide barriers: every thread widens its share of
    // tile it and signals convb; thread 0 issues tile it's MMAs once every share is
    // in and the epilogue of tile it - 2 has released the TMEM buffer; every thread
    // then runs the epilogue of tile it - 1.
    bool aborted = __syncthreads_or(!ok);
    int it = 0;
    for (; !aborted; ++it) {
        const int tile = tile_of(it);
        const bool have = tile < ntiles;
        if (have) {
            const int stage = it % kIdxStages;
            const int b = it & 1;
            if (!mbar_wait(&full[stage], (it / kIdxStages) & 1, p.err)) {
                aborted = true;
                break;
            }
            if (qa < qb) my_scl[b * kKeyTile + row] = scaled ? sc_s[stage * kKeyTile + row] : 1.0f;
            uint32_t a_addr;
            if constexpr (FP8) {
                // Widen 128 x 64 E4M3 codes to bf16 (exact) in the 128B-swizzled layout.
                const uint8_t* raw = ring + stage * raw_bytes;
                uint8_t* dst = cvt + b * kTileBytesBf16;
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int chunk = tid + rr * kThreads;
                    const int kr = chunk >> 2, piece = chunk & 3;
                    const uint4 v = *reinterpret_cast<const uint4*>(raw + kr * 64 + piece * 16);
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                    uint32_t o[8];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        o[2 * i] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w4[i] & 0xFFFFu));
                        o[2 * i + 1] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w4[i] >> 16));
                    }
                    const int c0 = (2 * piece) ^ (kr & 7), c1 = (2 * piece + 1) ^ (kr & 7);
                    *reinterpret_cast<uint4*>(dst + kr * 128 + c0 * 16) = make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4*>(dst + kr * 128 + c1 * 16) = make_uint4(o[4], o[5], o[6], o[7]);
                }
                fence_proxy_async_smem();
                a_addr = smem_u32(dst);
            } else {
                a_addr = smem_u32(ring + stage * raw_bytes);
            }
            mbar_arrive(&convb[b]);   // this thread is done with the raw stage (scale copy, widening)
            if (tid == 0) {
                bool okw = true;
                okw = mbar_wait(&convb[b], (it >> 1) & 1, p.err);
                if (okw && it >= 2) okw = mbar_wait(&tfree[b], ((it >> 1) - 1) & 1, p.err);
                if (okw) {
                    tc_fence_after();
                    const uint64_t adesc = umma_desc_sw128(a_addr);
#pragma unroll
                    for (int k = 0; k < kDI / 16; ++k)
                        tc_mma_bf16(tmem + b * 128, adesc + 2 * k, bdesc + 2 * k, idesc, k > 0 ? 1u : 0u);
                    tc_commit(&mmab[b]);
                    ++mma_issued;
                    if constexpr (FP8) {   // every share of the raw tile is consumed: refill its stage now
                        const int next = tile_of(it + kIdxStages);
                        if (next < ntiles) {
                            load_tile(stage, next);
                            ++issued;
                        }
                    }
                } else {
                    aborted = true;
                }
            }
            if (aborted) break;
        }
        if (it > 0) {
            if (!epilogue(it - 1)) {
                aborted = true;
                break;
            }
            if (tid == 0) mma_done = it;
            if constexpr (!FP8) {   // the MMAs of local tile it - 1 are complete: refill its stage
                const int next = tile_of(it - 1 + kIdxStages);
                if (tid == 0 && next < ntiles) {
                    load_tile((it - 1) % kIdxStages, next);
                    ++issued;
                }
            }
        }
        if (!have) break;
    }
    // A wait that ran out (error bit set) ends the loop for that thread; the others
    // run into bounded waits and stop too.  Copies and MMAs still in flight land
    // before the shared memory and TMEM are reused.
    aborted = __syncthreads_or(aborted);
    if (aborted && tid == 0) {
        mbar_wait(setup, 0, p.err);
        for (int k = it; k < issued; ++k) mbar_wait(&full[k % kIdxStages], (k / kIdxStages) & 1, p.err);
        for (int e = mma_done; e < mma_issued; ++e) mbar_wait(&mmab[e & 1], (e >> 1) & 1, p.err);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }

    // This block's key range of each query's visible scores (slot [block][t]).
#pragma unroll
    for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            klo[u] = min(klo[u], __shfl_xor_sync(0xffffffffu, klo[u], o));
            khi[u] = max(khi[u], __shfl_xor_sync(0xffffffffu, khi[u], o));
        }
    }
    // scratch[0..31]: lo of (query t, quad) at t*4 + quad; scratch[32..63]: hi.
    if (lane == 0)
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (qa + u < qb) {
                scratch[(qa + u) * 4 + quad] = klo[u];
                scratch[32 + (qa + u) * 4 + quad] = khi[u];
            }
    __syncthreads();
    if (tid < kMaxT && p.mm != nullptr) {
        uint32_t lo = 0xFFFFFFFFu, hi = 0u;
        if (tid < T)
            for (int q = 0; q < 4; ++q) {
                lo = min(lo, scratch[tid * 4 + q]);
                hi = max(hi, scratch[32 + tid * 4 + q]);
            }
        p.mm[(int64_t)blockIdx.x * kMaxT + tid] = make_uint2(lo, hi);
    }
    // Positions no query can see (s >= n_max): -inf, as the stage contract states.
    const int64_t tail0 = (int64_t)ntiles * kKeyTile;
    for (int64_t s = tail0 + (int64_t)blockIdx.x * kThreads + tid; s < p.L; s += (int64_t)gridDim.x * kThreads)
        for (int tt = 0; tt < T; ++tt) p.scores[(int64_t)tt * p.ld + s] = -INFINITY;
    __syncthreads();
}

// Phase 1 for caller-provided scores: each block's key range per query.
__device__ void phase_ranges(const StepParams& p, uint32_t* scratch)
{
    for (int i = blockIdx.x * kThreads + threadIdx.x; i < p.zero_words; i += gridDim.x * kThreads) p.zero[i] = 0u;
    for (int t = 0; t < p.T; ++t) {
        const int n = query_pos(p, t) + 1;
        uint32_t lo = 0xFFFFFFFFu, hi = 0u;
        const float* row = p.scores + (int64_t)t * p.ld;
        for (int s = blockIdx.x * kThreads + threadIdx.x; s < n; s += gridDim.x * kThreads) {
            const uint32_t k = score_key(__ldcg(row + s));
            lo = min(lo, k);
            hi = max(hi, k);
        }
        block_minmax(lo, hi, scratch);
        if (threadIdx.x == 0) p.mm[(int64_t)blockIdx.x * kMaxT + t] = make_uint2(lo, hi);
    }
    for (int t = p.T + threadIdx.x; t < kMaxT; t += kThreads)
        p.mm[(int64_t)blockIdx.x * kMaxT + t] = make_uint2(0xFFFFFFFFu, 0u);
}

// ==================================================================================
// Phases 2-4: causal top-k by radix select over the query's own key range.
// Work items are (query t, chunk c): positions [c*S, min((c+1)*S, n_t)); a block
// has at most one.  A chunk that fits is bulk-copied into shared memory once
// (phase 2) and stays there, as order-preserving keys, until phase 4; a longer
// one streams through a ring of bulk-copied tiles in each phase.  Phase 3 lists
// only the keys inside the threshold bin (few) and counts the keys above it per
// chunk; from those, every chunk block finds the exact threshold and its own
// offset in the output, then compacts its positions in order.
// ==================================================================================
constexpr int kChunkSmem = 32768;        // scores of one chunk kept in shared memory (128 KiB)
constexpr int kStreamStages = 8;         // ring of score tiles for longer chunks
constexpr int kStreamTile = 4096;        // scores per tile (16 KiB)
constexpr int kStreamBar = 32;           // first of the ring's mbarriers
constexpr int kStageCap = 8192;          // candidates phase 3 stages in shared memory before a flush
constexpr int kWork = kChunkSmem * 4;    // shared-memory offset of the region after the chunk
static_assert(kStreamStages * kStreamTile <= kChunkSmem, "the ring fits the chunk region");
static_assert(kChunkSmem * 4 + kStageCap * 8 <= kDataBytes, "chunk + candidate staging fit");
static_assert(kChunkSmem * 4 + kHistBins * 4 <= kDataBytes, "chunk + histogram fit");
static_assert(kStreamBar + kStreamStages <= kBarSlots, "ring mbarriers fit");

// Streams row[s0, s1) through the ring: for tile j, f(tile, a, c) runs on all
// threads with tile[0, c) = the scores of positions a .. a + c - 1.  `seq`
// counts the tiles this block has streamed so far (it keeps each stage's
// mbarrier parity in step across calls).  False if a wait ran out (error bit
// set; the copies still in flight are waited for before returning).
template <typename F>
__device__ bool stream_scores(const float* row, int s0, int s1, float* ring, uint64_t* full, uint32_t& seq,
                              uint32_t* err, F f)
{
    const int ntiles = s1 > s0 ? (s1 - s0 + kStreamTile - 1) / kStreamTile : 0;
    auto issue = [&](int j) {
        const int a = s0 + j * kStreamTile;
        const int c = min(kStreamTile, s1 - a);
        const uint32_t bytes = static_cast<uint32_t>((c + 3) & ~3) * 4u;   // rows have a stride of 4k scores
        const uint32_t st = (seq + j) % kStreamStages;
        mbar_arrive_expect_tx(&full[st], bytes);
        bulk_g2s(ring + st * kStreamTile, row + a, bytes, &full[st]);
    };
    fence_proxy_async_smem();   // earlier generic writes to the ring region come first
    __syncthreads();
    if (threadIdx.x == 0)
        for (int j = 0; j < min(ntiles, kStreamStages); ++j) issue(j);
    int j = 0;
    bool ok = true;
    for (; j < ntiles; ++j) {
        const uint32_t g = seq + j, st = g % kStreamStages;
        if (!__syncthreads_and(mbar_wait(&full[st], (g / kStreamStages) & 1u, err))) {
            ok = false;
            break;
        }
        const int a = s0 + j * kStreamTile;
        f(ring + st * kStreamTile, a, min(kStreamTile, s1 - a));
        __syncthreads();
        if (threadIdx.x == 0 && j + kStreamStages < ntiles) issue(j + kStreamStages);
    }
    if (!ok && threadIdx.x == 0)   // drain what is still in flight (bounded waits)
        for (int k = j; k < min(ntiles, j + kStreamStages); ++k) {
            const uint32_t g = seq + k;
            mbar_wait(&full[g % kStreamStages], (g / kStreamStages) & 1u, err);
        }
    seq += ntiles;
    __syncthreads();
    return ok;
}

struct Item {
    int t, c, s0, s1, n;
};

__device__ __forceinline__ Item topk_item(const StepParams& p, int i)
{
    Item it;
    it.t = i / p.nchunk;
    it.c = i % p.nchunk;
    int pos_t = 0;
#pragma unroll
    for (int k = 0; k < kMaxT; ++k)
        if (k == it.t) pos_t = query_pos(p, k);
    it.n = pos_t + 1;
    it.s0 = min(it.n, it.c * p.chunk);
    it.s1 = min(it.n, it.s0 + p.chunk);
    return it;
}

// Key range [lo, hi] of query t from the per-block ranges of phase 1.
__device__ void query_range(const StepParams& p, int t, uint32_t& lo, uint32_t& hi, uint32_t* scratch)
{
    lo = 0xFFFFFFFFu;
    hi = 0u;
    for (int b = threadIdx.x; b < p.mm_slots; b += kThreads) {
        const uint2 v = __ldcg(p.mm + (int64_t)b * kMaxT + t);
        lo = min(lo, v.x);
        hi = max(hi, v.y);
    }
    block_minmax(lo, hi, scratch);
}

// Per query: threshold bin [cut, ctop] and #(keys > ctop).
struct Cut {
    uint32_t cut, ctop, above;
};

__device__ void phase_hist(const StepParams& p, uint8_t* smem, uint64_t* bar, uint64_t* ring_full, uint32_t& seq,
                           uint32_t* scratch)
{
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem);                       // [kChunkSmem] (or the ring)
    uint32_t* h = reinterpret_cast<uint32_t*>(smem + kWork);                  // [kHistBins]
    for (int r = 0;; ++r) {
        const int i = item_of(r);
        if (i >= p.T * p.nchunk) break;
        const Item it = topk_item(p, i);
        if (it.n <= p.topk || it.s0 >= it.s1) continue;
        uint32_t lo, hi;
        query_range(p, it.t, lo, hi, scratch);
        const int shift = range_shift(lo, hi);
        const float* row = p.scores + (int64_t)it.t * p.ld;
        const int cnt = it.s1 - it.s0;
        const int c4 = (cnt + 3) & ~3;   // rows have a stride that is a multiple of 4 scores
        const bool in_smem = r == 0 && c4 <= kChunkSmem;   // a block's first item stays in smem
        if (in_smem) {
            fence_proxy_async_smem();
            __syncthreads();
            if (threadIdx.x == 0) {
                mbar_arrive_expect_tx(bar, static_cast<uint32_t>(c4) * 4u);
                bulk_g2s(keys, row + it.s0, static_cast<uint32_t>(c4) * 4u, bar);
            }
        }
        for (int b = threadIdx.x; b < kHistBins; b += kThreads) h[b] = 0u;
        if (in_smem) {
            const bool ok = mbar_wait(bar, 0, p.err);   // this barrier completes once per launch
            if (!__syncthreads_and(ok)) return;
            for (int j = threadIdx.x; j < cnt; j += kThreads) {
                const uint32_t k = score_key(__uint_as_float(keys[j]));
                keys[j] = k;
                atomicAdd(&h[(k - lo) >> shift], 1u);
            }
        } else {
            const bool ok = stream_scores(row, it.s0, it.s1, reinterpret_cast<float*>(keys), ring_full, seq, p.err,
                                          [&](const float* tile, int, int c) {
                                              for (int j = threadIdx.x; j < c; j += kThreads)
                                                  atomicAdd(&h[(score_key(tile[j]) - lo) >> shift], 1u);
                                          });
            if (!ok) return;
        }
        __syncthreads();
        uint32_t* gh = p.hist + (int64_t)it.t * kHistBins;
        for (int b = threadIdx.x; b < kHistBins; b += kThreads)
            if (h[b]) atomicAdd(gh + b, h[b]);
        __syncthreads();
    }
}

// The threshold bin of query t from its histogram (read with coalesced loads
// into h, shared memory).
__device__ Cut query_cut(const StepParams& p, int t, uint32_t* h, uint32_t* res, uint32_t* scratch)
{
    uint32_t lo, hi;
    query_range(p, t, lo, hi, scratch);
    const int shift = range_shift(lo, hi);
    const uint32_t* gh = p.hist + (int64_t)t * kHistBins;
    {
        uint32_t v[kHistBins / kThreads];   // every load in flight before the first use
#pragma unroll
        for (int i = 0; i < kHistBins / kThreads; ++i) v[i] = __ldcg(gh + threadIdx.x + i * kThreads);
#pragma unroll
        for (int i = 0; i < kHistBins / kThreads; ++i) h[threadIdx.x + i * kThreads] = v[i];
    }
    __syncthreads();
    find_from_top<kHistBins>(h, static_cast<uint32_t>(p.topk), res, scratch);
    Cut cu{lo, hi, 0u};
    if (res[2]) {
        cu.cut = lo + (res[0] << shift);
        cu.ctop = bin_top(cu.cut, shift, hi);
        cu.above = res[1];
    } else if (threadIdx.x == 0) {   // histogram and scores disagree: cannot happen for consistent input
        atomicOr(p.err, ERR_TOPK_STATE);
    }
    __syncthreads();
    return cu;
}

// Phase 3: every key >= cut (the threshold bin and above) goes to the query's
// candidate list with its position; the keys above the bin are also counted per
// chunk.
// Candidates are staged in shared memory (one shared atomic per warp step) and
// flushed to the list with one global atomic per flush; nothing downstream
// depends on the list's order.
__device__ void phase_extract(const StepParams& p, uint8_t* smem, uint64_t* ring_full, uint32_t& seq, uint32_t* res,
                              uint32_t* scratch)
{
    const uint32_t* keys = reinterpret_cast<const uint32_t*>(smem);             // resident chunk (phase 2)
    uint2* stage = reinterpret_cast<uint2*>(smem + kWork);                       // [kStageCap]
    __shared__ uint32_t nstage, flush_at;
    for (int r = 0;; ++r) {
        const int i = item_of(r);
        if (i >= p.T * p.nchunk) break;
        const Item it = topk_item(p, i);
        if (it.n <= p.topk) continue;
        const Cut cu = query_cut(p, it.t, reinterpret_cast<uint32_t*>(smem + kWork), res, scratch);
        if (it.c == 0 && threadIdx.x == 0)
            reinterpret_cast<uint4*>(p.cuts)[it.t] = make_uint4(cu.cut, cu.ctop, cu.above, 0u);
        if (threadIdx.x == 0) nstage = 0;
        __syncthreads();
        uint2* list = p.list + (int64_t)it.t * p.list_ld;
        // Move the staged candidates to the list (all threads; nstage is uniform here).
        auto flush = [&]() {
            const uint32_t n = min(nstage, static_cast<uint32_t>(kStageCap));
            if (n == 0) return;
            if (threadIdx.x == 0) flush_at = atomicAdd(p.list_n + it.t, n);
            __syncthreads();
            const uint32_t at = flush_at;
            for (uint32_t j = threadIdx.x; j < n; j += kThreads) list[at + j] = stage[j];
            __syncthreads();
            if (threadIdx.x == 0) nstage = 0;
            __syncthreads();
        };
        uint32_t above = 0;
        const int cnt = it.s1 - it.s0;
        const bool resident = r == 0 && ((cnt + 3) & ~3) <= kChunkSmem;
        // Keys of positions a .. a + c - 1 (at most kStreamTile of them).
        auto take = [&](auto key_at, int a, int c) {
            if (nstage + static_cast<uint32_t>(c) > static_cast<uint32_t>(kStageCap)) flush();
            for (int j0 = 0; j0 < c; j0 += kThreads) {
                const int j = j0 + threadIdx.x;
                const uint32_t k = j < c ? key_at(j) : 0u;
                above += j < c && k > cu.ctop;
                warp_append(j < c && k >= cu.cut, make_uint2(k, static_cast<uint32_t>(a + j)), stage, &nstage,
                            kStageCap);
            }
        };
        if (cnt > 0) {
            if (resident) {
                for (int a = 0; a < cnt; a += kStreamTile) {
                    take([&](int j) { return keys[a + j]; }, it.s0 + a, min(kStreamTile, cnt - a));
                    __syncthreads();
                }
            } else {
                const float* row = p.scores + (int64_t)it.t * p.ld;
                const bool ok = stream_scores(row, it.s0, it.s1, reinterpret_cast<float*>(smem), ring_full, seq,
                                              p.err, [&](const float* tile, int a, int c) {
                                                  take([&](int j) { return score_key(tile[j]); }, a, c);
                                              });
                if (!ok) return;
            }
            flush();
        }
        above = block_sum(above, scratch);
        if (threadIdx.x == 0) p.above[(int64_t)it.t * kMaxChunksStep + it.c] = above;
    }
}

// Radix select over n values read through get(j) (only those in [lo, hi] count),
// `need` of them still to find from the top.  On return lo == hi is the need-th
// largest value and need = how many entries equal to it are to be taken.
template <typename Get>
__device__ void radix_select(Get get, uint32_t n, uint32_t& lo, uint32_t& hi, uint32_t& need, uint32_t* h,
                             uint32_t* res, uint32_t* scratch, uint32_t* err)
{
#pragma unroll 1
    for (int pass = 0; pass < 4 && lo != hi; ++pass) {
        const int shift = range_shift(lo, hi);
        for (int b = threadIdx.x; b < kHistBins; b += kThreads) h[b] = 0u;
        __syncthreads();
        for (uint32_t j = threadIdx.x; j < n; j += kThreads) {
            const uint32_t k = get(j);
            if (k >= lo && k <= hi) atomicAdd(&h[(k - lo) >> shift], 1u);
        }
        __syncthreads();
        find_from_top<kHistBins>(h, need, res, scratch);
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
}

// The need-th largest of the n values v[0..n) gathered in shared memory: radix
// select with 256 bins over their own range [min, max] (no pass at all when the
// values are equal).  Returns the value; `need` becomes how many entries equal
// to it are to be taken.
constexpr int kSmallBins = 256;

__device__ uint32_t small_select(const uint32_t* v, uint32_t n, uint32_t& need, uint32_t* h, uint32_t* res,
                                 uint32_t* scratch, uint32_t* err)
{
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (uint32_t j = threadIdx.x; j < n; j += kThreads) {
        lo = min(lo, v[j]);
        hi = max(hi, v[j]);
    }
    block_minmax(lo, hi, scratch);
#pragma unroll 1
    for (int pass = 0; pass < 4 && lo != hi; ++pass) {
        const int bits = 32 - __clz(hi - lo);
        const int shift = bits > 8 ? bits - 8 : 0;
        h[threadIdx.x] = 0u;   // kSmallBins == kThreads
        __syncthreads();
        for (uint32_t j = threadIdx.x; j < n; j += kThreads) {
            const uint32_t x = v[j];
            if (x >= lo && x <= hi) atomicAdd(&h[(x - lo) >> shift], 1u);
        }
        __syncthreads();
        find_from_top<kSmallBins>(h, need, res, scratch);
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
    return lo;
}

// The need-th largest of the n values v[0..n) in shared memory (n small): each
// thread ranks its values against all of them, one step.  Returns the value;
// `need` becomes how many entries equal to it are to be taken.
constexpr int kRankSel = 64;

__device__ uint32_t rank_select(const uint32_t* v, uint32_t n, uint32_t& need, uint32_t* res, uint32_t* err)
{
    if (threadIdx.x == 0) res[2] = 0;
    __syncthreads();
    for (uint32_t j = threadIdx.x; j < n; j += kThreads) {
        const uint32_t x = v[j];
        uint32_t gt = 0, eq = 0, eq_before = 0;
        for (uint32_t q = 0; q < n; ++q) {
            const uint32_t y = v[q];
            gt += y > x;
            eq += y == x;
            eq_before += (y == x) && q < j;
        }
        // the first copy (lowest index) of the value that holds the need-th place reports it
        if (eq_before == 0 && gt < need && gt + eq >= need) {
            res[0] = x;
            res[1] = gt;
            res[2] = 1;
        }
    }
    __syncthreads();
    uint32_t x = 0u;
    if (res[2]) {
        x = res[0];
        need -= res[1];
    } else if (threadIdx.x == 0) {
        atomicOr(err, ERR_TOPK_STATE);
    }
    __syncthreads();
    return x;
}

__device__ __forceinline__ uint32_t exact_select(uint32_t* v, uint32_t n, uint32_t& need, uint32_t* h, uint32_t* res,
                                                 uint32_t* scratch, uint32_t* err)
{
    return n <= static_cast<uint32_t>(kRankSel) ? rank_select(v, n, need, res, err)
                                                : small_select(v, n, need, h, res, scratch, err);
}

// Phase 4: ordered emission, one item per (query t, chunk c).  The block reads
// the query's threshold-bin candidates (few) and the per-chunk counts of keys
// above the bin, finds the exact threshold tau (the topk-th largest key) and the
// tie cut pcut (keys equal to tau are taken at positions <= pcut), and so its
// first output slot; then it marks the selected positions of its chunk (all in
// the list) in a bitmap and writes them in ascending order.  More than kInCap
// candidates (heavy ties) take radix selects over the list in global memory and
// an ordered compaction of the chunk's keys: each warp owns 512 consecutive
// positions of a tile, counts them with ballots and writes them after the warps
// before it.
constexpr int kInCap = 3584;             // candidates gathered in shared memory
constexpr int kChunkWords = 16384;       // bitmap words of a streamed chunk (2^19 positions)
static_assert(kChunkWords * 4 <= kWork, "the bitmap fits below the list");
static_assert(kWork + kHistBins * 4 + kInCap * 12 <= kDataBytes, "emission buffers fit");

__device__ void phase_emit(const StepParams& p, uint8_t* smem, uint64_t* ring_full, uint32_t& seq, uint32_t* res,
                           uint32_t* scratch)
{
    const uint32_t* keys = reinterpret_cast<const uint32_t*>(smem);   // resident chunk (phase 2)
    uint32_t* h = reinterpret_cast<uint32_t*>(smem + kWork);          // [kHistBins] select bins
    uint2* in = reinterpret_cast<uint2*>(h + kHistBins);              // [kInCap] (key, position)
    uint32_t* vals = reinterpret_cast<uint32_t*>(in + kInCap);        // [kInCap]
    __shared__ uint32_t nval;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kSeg = kStreamTile / kWarps;                         // positions per warp and tile
    for (int r = 0;; ++r) {
        const int i = item_of(r);
        if (i >= p.T * p.nchunk) break;
        const Item it = topk_item(p, i);
        int32_t* sel = p.sel + (int64_t)it.t * p.sel_ld;
        if (it.n <= p.topk) {   // everything visible is selected
            for (int s = it.s0 + tid; s < it.s1; s += kThreads) sel[s] = s;
            if (it.c == 0)
                for (int j = it.n + tid; j < p.topk; j += kThreads) sel[j] = -1;
            continue;
        }
        const int cnt = it.s1 - it.s0;
        if (cnt <= 0) continue;
        const uint32_t m = __ldcg(p.list_n + it.t);
        const uint4 cq = __ldcg(reinterpret_cast<const uint4*>(p.cuts) + it.t);
        const Cut cu{cq.x, cq.y, cq.z};
        const uint2* glist = p.list + (int64_t)it.t * p.list_ld;
        const uint32_t* above = p.above + (int64_t)it.t * kMaxChunksStep;
        // keys above the bin in the chunks before this one
        uint32_t before = 0;
        for (int c = tid; c < it.c; c += kThreads) before += __ldcg(above + c);
        const bool fits = m <= static_cast<uint32_t>(kInCap);
        if (fits)
            for (uint32_t j0 = 0; j0 < m; j0 += 8 * kThreads) {   // eight loads in flight per thread
                uint2 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint32_t j = j0 + u * kThreads + tid;
                    v[u] = j < m ? __ldcg(glist + j) : make_uint2(0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint32_t j = j0 + u * kThreads + tid;
                    if (j < m) in[j] = v[u];
                }
            }
        if (tid == 0) nval = 0;
        __syncthreads();
        uint32_t nin = 0;   // keys inside the threshold bin, gathered in vals
        if (fits) {
            for (uint32_t j0 = 0; j0 < m; j0 += kThreads) {
                const uint32_t j = j0 + tid;
                const uint32_t k = j < m ? in[j].x : 0xFFFFFFFFu;
                warp_append(j < m && k <= cu.ctop, k, vals, &nval, kInCap);
            }
            __syncthreads();
            nin = nval;
            __syncthreads();
            if (tid == 0) nval = 0;
        }
        stamp(p, 12);

        uint32_t need = static_cast<uint32_t>(p.topk) - cu.above;
        uint32_t tau, pcut = 0xFFFFFFFFu;   // selected: key > tau, or key == tau and position <= pcut
        if (fits) {
            tau = exact_select(vals, nin, need, h, res, scratch, p.err);   // ends with a barrier
            const uint32_t rties = need;
            for (uint32_t j0 = 0; j0 < m; j0 += kThreads) {   // ~position of the ties: largest = lowest
                const uint32_t j = j0 + tid;
                const uint2 v = j < m ? in[j] : make_uint2(0u, 0u);
                warp_append(j < m && v.x == tau, ~v.y, vals, &nval, kInCap);
            }
            __syncthreads();
            const uint32_t e = nval;
            if (rties < e) pcut = ~exact_select(vals, e, need, h, res, scratch, p.err);
            for (uint32_t j = tid; j < m; j += kThreads) {
                const uint2 v = in[j];
                before += static_cast<int>(v.y) < it.s0 && v.x <= cu.ctop && (v.x > tau || (v.x == tau && v.y <= pcut));
            }
        } else {
            uint32_t lo = cu.cut, hi = cu.ctop;
            radix_select([&](uint32_t j) { return __ldcg(glist + j).x; }, m, lo, hi, need, h, res, scratch, p.err);
            tau = lo;   // (keys above ctop in the list fall outside [lo, hi] and are not counted)
            uint32_t e = 0, plo = 0xFFFFFFFFu, phi = 0u;
            for (uint32_t j = tid; j < m; j += kThreads) {
                const uint2 v = __ldcg(glist + j);
                if (v.x == tau) {
                    ++e;
                    plo = min(plo, ~v.y);
                    phi = max(phi, ~v.y);
                }
            }
            e = block_sum(e, scratch);
            block_minmax(plo, phi, scratch);
            if (need < e) {
                radix_select(
                    [&](uint32_t j) {
                        const uint2 v = __ldcg(glist + j);
                        return v.x == tau ? ~v.y : 0u;
                    },
                    m, plo, phi, need, h, res, scratch, p.err);
                pcut = ~plo;
            }
            for (uint32_t j = tid; j < m; j += kThreads) {
                const uint2 v = __ldcg(glist + j);
                before += static_cast<int>(v.y) < it.s0 && v.x <= cu.ctop && (v.x > tau || (v.x == tau && v.y <= pcut));
            }
        }
        uint32_t out = block_sum(before, scratch);   // this chunk's first output slot
        stamp(p, 13);
        const uint32_t topk = static_cast<uint32_t>(p.topk);
        auto emit_tile = [&](auto key_at, int a, int c) {
            auto chosen = [&](int j) {
                if (j >= c) return false;
                const uint32_t k = key_at(j);
                return k > tau || (k == tau && static_cast<uint32_t>(a + j) <= pcut);
            };
            uint32_t wc = 0;
#pragma unroll 4
            for (int u = 0; u < kSeg / 32; ++u)
                wc += __popc(__ballot_sync(0xffffffffu, chosen(warp * kSeg + u * 32 + lane)));
            if (lane == 0) scratch[warp] = wc;
            __syncthreads();
            uint32_t wo = out, tot = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const uint32_t x = scratch[w];
                wo += w < warp ? x : 0u;
                tot += x;
            }
            __syncthreads();
            const uint32_t wend = wo + wc;
            for (int u = 0; u < kSeg / 32 && wo < wend; ++u) {
                const int j = warp * kSeg + u * 32 + lane;
                const bool s = chosen(j);
                const uint32_t bal = __ballot_sync(0xffffffffu, s);
                const uint32_t o = wo + __popc(bal & ((1u << lane) - 1u));
                if (s && o < topk) sel[o] = a + j;
                wo += __popc(bal);
            }
            out += tot;
        };
        const int R = ((cnt + 31) / 32 + kThreads - 1) / kThreads;   // bitmap words per thread
        if (fits && R * kThreads <= kChunkWords) {
            // Bitmap of the chunk's selected positions, transposed: thread i owns the
            // R consecutive words [i*R, (i+1)*R), its k-th word at k*256 + i.
            uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem);
            for (int w = tid; w < R * kThreads; w += kThreads) bitmap[w] = 0u;
            __syncthreads();
            for (uint32_t j = tid; j < m; j += kThreads) {
                const uint2 v = in[j];
                const int q = static_cast<int>(v.y);
                if (q >= it.s0 && q < it.s1 && (v.x > tau || (v.x == tau && v.y <= pcut))) {
                    const uint32_t rel = static_cast<uint32_t>(q - it.s0), w = rel >> 5, owner = w / R;
                    atomicOr(&bitmap[(w - owner * R) * kThreads + owner], 1u << (rel & 31));
                }
            }
            __syncthreads();
            uint32_t c1 = 0;
            for (int k = 0; k < R; ++k) c1 += __popc(bitmap[k * kThreads + tid]);
            uint32_t total;
            uint32_t o = out + block_excl_scan(c1, total, scratch);
            for (int k = 0; k < R && c1; ++k) {
                uint32_t b = bitmap[k * kThreads + tid];
                const int base = it.s0 + ((tid * R + k) << 5);
                while (b) {
                    const int bit = __ffs(b) - 1;
                    b &= b - 1;
                    if (o < topk) sel[o] = base + bit;
                    ++o;
                    --c1;
                }
            }
            out += total;
        } else if (r == 0 && ((cnt + 3) & ~3) <= kChunkSmem) {
            for (int a = 0; a < cnt; a += kStreamTile)
                emit_tile([&](int j) { return keys[a + j]; }, it.s0 + a, min(kStreamTile, cnt - a));
        } else {
            const float* row = p.scores + (int64_t)it.t * p.ld;
            const bool ok = stream_scores(row, it.s0, it.s1, reinterpret_cast<float*>(smem), ring_full, seq, p.err,
                                          [&](const float* tile, int a, int c) {
                                              emit_tile([&](int j) { return score_key(tile[j]); }, a, c);
                                          });
            if (!ok) return;
        }
        if (tid == 0 && (out > topk || (it.s1 == it.n && out != topk))) atomicOr(p.err, ERR_TOPK_STATE);
        __syncthreads();
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
        int pos_t = 0;
#pragma unroll
        for (int k = 0; k < kMaxT; ++k)
            if (k == t) pos_t = query_pos(p, k);
        const int cnt = min(pos_t + 1, p.window);
        p.sel[(int64_t)t * p.sel_ld + j] = j < cnt ? pos_t + 1 - cnt + j : -1;
    }
}

// ==================================================================================
// Phase 5: sparse attention per (query t, row split).  Warp 4 gathers whole
// 2 KiB token rows (K then V of the 4 groups) by bulk async copy into a 6-stage
// ring of 16-row tiles; warp g < 4 owns KV group g, i.e. query heads
// 16g .. 16g+15 -- the 16 rows of an m16n8k16 tile, so nothing is padded.
// Online softmax in the exp2 domain; the partial (max, sum, output) of every
// head goes to global memory for phase 6.
// ==================================================================================
__device__ void phase_attend(const StepParams& p, uint8_t* smem, uint64_t* bars)
{
    uint8_t* ring = smem;
    int32_t* rowidx = reinterpret_cast<int32_t*>(smem + kAttStages * kTileRows * kPitch);   // [stage][16]
    int32_t* sel_s = rowidx + kAttStages * kTileRows;
    uint64_t* full = bars + 8;
    uint64_t* empty = full + kAttStages;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, c = lane & 3;
    constexpr int kConsumers = 4;
    const float sm_scale = kLog2e * rsqrtf(static_cast<float>(kD));

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
        int pos_t = 0;
#pragma unroll
        for (int k = 0; k < kMaxT; ++k)
            if (k == t) pos_t = query_pos(p, k);
        const int rows_t = min(p.rows, pos_t + 1);
        const int r0 = split * p.rows_per_split;
        const int r1 = min(r0 + p.rows_per_split, rows_t);
        const int ntile = r1 > r0 ? (r1 - r0 + kTileRows - 1) / kTileRows : 0;

        bool failed = false;
        float oacc[16][4];
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) oacc[k][0] = oacc[k][1] = oacc[k][2] = oacc[k][3] = 0.f;

        if (warp == kConsumers) {
            // producer: validate the selected rows, gather them whole
            const int32_t* selrow = p.sel + (int64_t)t * p.sel_ld + r0;
            {
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
            if (tid == kConsumers * 32)
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
    }
}

// Phase 6: merge the splits of each (query, head) in split order.  Thread
// (g, d) sums splits g, g+4, ... for dims 2d, 2d+1; the four partial sums are
// then added in a fixed order.
// Phase 6 for one or two queries (many splits per head): one block per (query,
// head); four thread groups share the splits, with every split's (max, sum) in
// one load per thread and eight partial-output loads in flight per thread.
__device__ void phase_merge_block(const StepParams& p, uint8_t* smem, uint32_t* scratch)
{
    float* part = reinterpret_cast<float*>(smem);   // [4][128] partial sums + [4] denominators
    float* wsp = part + 4 * kD + 4;                 // [kMaxAttnItems] weight of each split
    const int items = p.T * kH;
    const int tid = threadIdx.x, grp = tid >> 6, d2 = tid & 63;
    for (int r = 0;; ++r) {
        const int i = item_of(r);
        if (i >= items) break;
        const int t = i / kH, h = i % kH;
        const float2* ml = p.pml + (int64_t)t * p.nsplit * kH + h;
        // (max, sum) of every split, one load per thread, then the running max
        float2 mv[kMaxAttnItems / kThreads];
#pragma unroll
        for (int u = 0; u < kMaxAttnItems / kThreads; ++u) {
            const int s = tid + u * kThreads;
            mv[u] = s < p.nsplit ? __ldcg(ml + (int64_t)s * kH) : make_float2(-INFINITY, 0.f);
        }
        float M = -INFINITY;
#pragma unroll
        for (int u = 0; u < kMaxAttnItems / kThreads; ++u) M = fmaxf(M, mv[u].x);
        float sink = -INFINITY;
        if (p.sink != nullptr) sink = p.sink[h] * kLog2e;
        M = fmaxf(M, sink);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        if ((tid & 31) == 0) scratch[tid >> 5] = __float_as_uint(M);
        __syncthreads();
        M = __uint_as_float(scratch[0]);
#pragma unroll
        for (int w = 1; w < kWarps; ++w) M = fmaxf(M, __uint_as_float(scratch[w]));
        // split weights (0 for a split without rows) and this thread's share of the denominator
        float den = 0.f;
#pragma unroll
        for (int u = 0; u < kMaxAttnItems / kThreads; ++u) {
            const int s = tid + u * kThreads;
            if (s < p.nsplit) {
                const float w = mv[u].x == -INFINITY ? 0.f : exp2f(mv[u].x - M);
                wsp[s] = w;
                den += w * mv[u].y;
            }
        }
        __syncthreads();
        // numerator: group g takes splits g, g+4, ...; eight loads in flight per thread
        float ax = 0.f, ay = 0.f;
        const float2* po = reinterpret_cast<const float2*>(p.po + ((int64_t)t * p.nsplit * kH + h) * kD) + d2;
        for (int s0 = grp; s0 < p.nsplit; s0 += 32) {
            float2 ov[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int s = s0 + 4 * u;
                ov[u] = (s < p.nsplit && wsp[s] > 0.f) ? __ldcg(po + (int64_t)s * kH * (kD / 2)) : make_float2(0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int s = s0 + 4 * u;
                const float w = s < p.nsplit ? wsp[s] : 0.f;
                ax = fmaf(w, ov[u].x, ax);
                ay = fmaf(w, ov[u].y, ay);
            }
        }
        part[grp * kD + 2 * d2] = ax;
        part[grp * kD + 2 * d2 + 1] = ay;
        den = block_sum_f(den, scratch);
        if (grp == 0) {
            float dd = den + ((p.sink != nullptr && M != -INFINITY) ? exp2f(sink - M) : 0.f);
            float x = 0.f, y = 0.f;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                x += part[g * kD + 2 * d2];
                y += part[g * kD + 2 * d2 + 1];
            }
            const float inv = dd > 0.f ? 1.0f / dd : 0.f;
            *reinterpret_cast<uint32_t*>(p.out + ((int64_t)t * kH + h) * kD + 2 * d2) = pack_bf16(x * inv, y * inv);
        }
        __syncthreads();
    }
}

// Phase 6 for three or more queries: one warp per item (query t, head h, half of
// the 128 dims): every split's (max, sum) with one load per lane and split, the
// running max and the denominator by warp shuffles, the weighted partial outputs
// with sixteen loads in flight per lane, all in a fixed order.  A sink joins the
// denominator with no value row.
constexpr int kMergeSplitsSmem = 512;      // split weights a warp keeps in shared memory (>= nsplit)
static_assert(kWarps * 2 * kMergeSplitsSmem * 4 <= kDataBytes, "merge weights fit");
static_assert(kMaxAttnItems <= kMergeSplitsSmem, "every split has a weight slot");

__device__ void phase_merge(const StepParams& p, uint8_t* smem, uint32_t* /*scratch*/)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* wsp = reinterpret_cast<float*>(smem) + warp * 2 * kMergeSplitsSmem;   // this warp's split weights
    float* lsp = wsp + kMergeSplitsSmem;                                            // and split sums
    constexpr int P = 2;                          // halves of the 128 dims per (t, h); two dims per lane
    const int items = p.T * kH * P;
    const int ns = p.nsplit;
    for (int i = blockIdx.x * kWarps + warp; i < items; i += gridDim.x * kWarps) {
        const int t = i / (kH * P), h = (i / P) % kH, part = i % P;
        const float2* ml = p.pml + (int64_t)t * ns * kH + h;
        float M = -INFINITY;
        for (int s0 = 0; s0 < ns; s0 += 32 * 4) {   // four (max, sum) loads in flight per lane
            float2 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int s = s0 + u * 32 + lane;
                v[u] = s < ns ? __ldcg(ml + (int64_t)s * kH) : make_float2(-INFINITY, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int s = s0 + u * 32 + lane;
                if (s < ns) {
                    wsp[s] = v[u].x;   // the split's max for now, its weight below
                    lsp[s] = v[u].y;
                }
                M = fmaxf(M, v[u].x);
            }
        }
        const float sink = p.sink != nullptr ? p.sink[h] * kLog2e : -INFINITY;
        M = fmaxf(M, sink);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float den = 0.f;
        for (int s = lane; s < ns; s += 32) {
            const float m = wsp[s];
            const float w = m == -INFINITY ? 0.f : exp2f(m - M);
            den += w * lsp[s];
            wsp[s] = w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        __syncwarp();
        // numerator for this lane's dims, splits in order, sixteen loads in flight
        const int d0 = part * (kD / P) + lane * 2;
        const float* po = p.po + ((int64_t)t * ns * kH + h) * kD + d0;
        float x0 = 0.f, x1 = 0.f;
        for (int s0 = 0; s0 < ns; s0 += 16) {
            float2 o[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int s = s0 + u;
                o[u] = (s < ns && wsp[s] > 0.f) ? __ldcg(reinterpret_cast<const float2*>(po + (int64_t)s * kH * kD))
                                                : make_float2(0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int s = s0 + u;
                const float w = s < ns ? wsp[s] : 0.f;
                x0 = fmaf(w, o[u].x, x0);
                x1 = fmaf(w, o[u].y, x1);
            }
        }
        const float dd = den + ((p.sink != nullptr && M != -INFINITY) ? exp2f(sink - M) : 0.f);
        const float inv = dd > 0.f ? 1.0f / dd : 0.f;
        *reinterpret_cast<uint32_t*>(p.out + ((int64_t)t * kH + h) * kD + d0) = pack_bf16(x0 * inv, x1 * inv);
        __syncwarp();
    }
}

// ==================================================================================
template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    step_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap smap, const StepParams p)
{
    // Query positions read from device memory (pos_dev), so that one CUDA graph of
    // the step serves every decode position.  A position outside [0, L) is clamped
    // and flagged.
    if (p.pos_dev != nullptr) {
        if (threadIdx.x < 32) {
            int v = 0;
            if (threadIdx.x < p.T) {
                v = __ldcg(p.pos_dev + threadIdx.x);
                if (v < 0 || v >= p.L) {
                    if (blockIdx.x == 0) atomicOr(p.err, ERR_BAD_POS);
                    v = min(max(v, 0), p.L - 1);
                }
            }
            if (threadIdx.x < kMaxT) g_qpos.pos[threadIdx.x] = v;
            int n = threadIdx.x < p.T ? v + 1 : 0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) n = max(n, __shfl_xor_sync(0xffffffffu, n, o));
            if (threadIdx.x == 0) g_qpos.n_max = n;
        }
        __syncthreads();
    }
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOffset);
    __shared__ uint32_t scratch[64];
    __shared__ uint32_t res[3];
    __shared__ int ok_s;
    __shared__ uint32_t tmem_slot;

    GridBarrier gb{p.bar_ctrl, p.err, gridDim.x, p.barrier_limit, p.barrier_extra};

    if (threadIdx.x == 0) {
        mbar_init(bars + 24, 1);
        for (int s = 0; s < kStreamStages; ++s) mbar_init(bars + kStreamBar + s, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Stamps (when tracing): 0 start, 1 indexer done, 2-3 histogram, 4-5 extract,
    // 6-7 emit, 8-9 attention, 10-11 merge (even: phase starts after its barrier).
    bool ok = true;
    uint32_t seq = 0;   // score tiles this block has streamed (phases 2-3)
    if (p.bar_ctrl != nullptr) gb.enter();
    stamp(p, 0);
    if (p.trace != nullptr && threadIdx.x == 0) p.trace[(int64_t)blockIdx.x * kTraceSlots + 28] = clock64();
    if (p.phases & kPhaseIndex) {
        phase_index<FP8>(kmap, smap, p, smem, bars, scratch, &tmem_slot);
    } else if (p.phases & kPhaseRanges) {
        phase_ranges(p, scratch);
    }
    stamp(p, 1);
    if (p.phases & kPhaseTopk) {
        ok = gb.sync(&ok_s);
        stamp(p, 2);
        if (ok) phase_hist(p, smem, bars + 24, bars + kStreamBar, seq, scratch);
        stamp(p, 3);
        ok = gb.sync(&ok_s) && ok;
        stamp(p, 4);
        if (ok) phase_extract(p, smem, bars + kStreamBar, seq, res, scratch);
        stamp(p, 5);
        ok = gb.sync(&ok_s) && ok;
        stamp(p, 6);
        if (ok) phase_emit(p, smem, bars + kStreamBar, seq, res, scratch);
        stamp(p, 7);
    }
    if (p.phases & kPhaseSelectPos) phase_select_pos(p);
    if (p.phases & kPhaseAttend) {
        if (p.phases & (kPhaseIndex | kPhaseTopk | kPhaseSelectPos)) ok = gb.sync(&ok_s) && ok;
        stamp(p, 8);
        if (ok) phase_attend(p, smem, bars);
        stamp(p, 9);
        ok = gb.sync(&ok_s) && ok;
        stamp(p, 10);
        if (ok) {
            if (p.T <= 2)
                phase_merge_block(p, smem, scratch);
            else
                phase_merge(p, smem, scratch);
        }
        stamp(p, 11);
    }
    if (p.bar_ctrl != nullptr) barrier_exit(p);
    if (p.trace != nullptr && threadIdx.x == 0) {
        p.trace[(int64_t)blockIdx.x * kTraceSlots + 29] = clock64();
        stamp(p, 30);
    }
}

bool g_configured[64][2] = {};

}  // namespace

int step_smem_bytes() { return kStepSmem; }

cudaError_t launch_step(const CUtensorMap* kmap, const CUtensorMap* smap, const StepParams& p, bool fp8,
                        cudaStream_t s)
{
    int dev = 0;
    cudaGetDevice(&dev);
    auto kern = fp8 ? step_kernel<true> : step_kernel<false>;
    if (dev >= 0 && dev < 64 && !g_configured[dev][fp8]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kStepSmem);
        if (e != cudaSuccess) return e;
        g_configured[dev][fp8] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kStepSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, *kmap, *smap, p);
}

int step_max_blocks(bool fp8)
{
    int dev = 0, sms = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    auto kern = fp8 ? step_kernel<true> : step_kernel<false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kStepSmem);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, kStepSmem) != cudaSuccess || n < 1) n = 1;
    cudaGetLastError();
    return sms * (n > 1 ? 1 : n);   // one block per SM
}

}  // namespace dsa
