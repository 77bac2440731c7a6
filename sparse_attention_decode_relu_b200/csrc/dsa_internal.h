// dsa_internal.h -- launchers and parameter blocks shared by the host side of
// libdsa (dsa_api.cu) and the kernel translation units.  Not part of the ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace dsa {

constexpr int kH = 64, kG = 4, kD = 128;   // backbone heads, KV groups, head dim
constexpr int kHI = 16, kDI = 64;          // indexer heads, indexer dim
constexpr int kMaxT = 8;
constexpr int kMaxTopk = 2048;
constexpr int kKeyTile = 128;              // keys per indexer tile
constexpr int kHistBins = 4096;            // first radix level: the top 12 bits of a score key
constexpr int kHistShift = 20;             // key >> kHistShift is the bin

constexpr int kMaxRowsPerSplit = 512;       // selected rows one attention work item gathers
constexpr int kMaxSplitsQ = 32;             // attention row splits per query
constexpr int kMinRowsPerSplit = 64;        // (so that topk <= 2048 rows make at most kMaxSplitsQ splits)
constexpr int kMaxChunksStep = 1024;        // top-k chunks per query (<= grid)
constexpr int kSegPerChunk = 8;             // candidate sub-segments per chunk (one per warp)
constexpr int kMaxSeg = kMaxChunksStep * kSegPerChunk;
constexpr int kMaxGrid = 1024;              // blocks of the step kernel
constexpr int kTraceSlots = 32;             // phase-boundary stamps per block

// Workspace control region.  Words (uint32) of the first 1024 bytes:
//   0          grid-barrier arrival count      (own 128-byte line)
//   32         exit count                      (own line)
//   64         launch epoch (never reset; selects the histogram buffer)
//   96 + t     extraction items of query t that are done
//   128 + t    query t's selection is written
//   160 + t    attention splits of query t that are done
// then two global histograms [2][kMaxT][kHistBins] u32.  Every word but the
// epoch is zero again when a launch ends; launch e uses histogram e & 1 and
// clears histogram (e + 1) & 1 for the next one.  The whole region must be zero
// before a workspace's first use.
constexpr int kCtrlWordExit = 32, kCtrlWordEpoch = 64, kCtrlWordArrive = 96, kCtrlWordReady = 128,
              kCtrlWordDone = 160, kCtrlWordBad = 192;
constexpr int kCtrlBytes = 1024;
constexpr int kHistWords = kMaxT * kHistBins;                 // one histogram buffer
constexpr int kWsCtrlBytes = kCtrlBytes + 2 * kHistWords * 4;  // must be zero before first use

constexpr long long kWaitLimitCycles = 2000000000LL;   // every spin gives up after this many SM clocks (~1 s)

// Phases of the step kernel.
enum : int {
    kPhaseIndex = 1,       // indexer scan (scores; with a workspace also the first radix histogram)
    kPhaseHistScores = 2,  // first radix histogram of caller-provided scores
    kPhaseTopk = 4,        // candidate extraction, per-query selection
    kPhaseAttend = 8,      // split attention + merge
    kPhaseSelectPos = 16,  // selection by position: the last `window` visible positions
};

struct StepParams {
    int32_t phases;
    int32_t grid;            // blocks (one per SM, all co-resident)
    int32_t T, L, n_max, topk;
    int32_t pos[kMaxT];
    const int32_t* pos_dev;  // nullptr, or pos [T] in device memory read at launch (then n_max = L here)
    // indexer
    const uint16_t* q_idx;   // [T][16][64] bf16
    const float* w;          // [T][16]
    const float* scale;      // [L] or nullptr
    float* scores;           // [T][ld]
    int64_t ld;
    // top-k
    uint32_t* cuts;          // [kMaxT][4]: lowest candidate key, #keys above the selection range, its top key
    uint32_t* seg_n;         // [kMaxT][kMaxSeg] candidates per sub-segment
    uint2* list;             // [T][list_ld] (key, position): sub-segment (c, w) starts at c*chunk + w*chunk/8
    int64_t list_ld;         // candidate-list row stride (the workspace's, not the caller's score stride)
    int32_t chunk, nchunk;   // extraction items: nchunk chunks of `chunk` positions per query (chunk % 256 == 0)
    int32_t* sel;            // [T][sel_ld]
    int64_t sel_ld;
    // attention
    const uint16_t* q;       // [T][64][128] bf16
    const uint16_t* kv;      // [L][kv_ld] bf16
    int64_t kv_ld;
    int32_t rows;            // selected rows per query to read (= topk)
    int32_t rows_per_split;  // multiple of 16, <= kMaxRowsPerSplit
    int32_t nsplit;          // row splits per query, <= kMaxSplitsQ
    const float* sink;       // [64] or nullptr
    int32_t window;          // kPhaseSelectPos: positions selected per query (<= topk)
    float* po;               // [T][nsplit][64][128] partial outputs per (query, split)
    float2* pml;             // [T][nsplit][64] (max in log2 units, sum)
    uint16_t* out;           // [T][64][128] bf16
    // control
    unsigned long long* trace;   // [grid][kTraceSlots] globaltimer stamps at phase boundaries, or nullptr
    uint32_t* ctrl;          // workspace control region (kWsCtrlBytes), or nullptr (indexer stage alone)
    int64_t barrier_limit;   // SM clocks a wait between blocks spins before it gives up
    uint32_t barrier_extra;  // arrivals such a wait needs beyond the real ones (0; 1 = a block that never comes)
    uint32_t* err;
    int32_t hist_bound;      // the first radix histogram holds per-thread key maxima (a lower bound), not every key
    uint32_t* gmax;          // [T][gmax_ld] largest key of each 32-position group (0: none visible), or nullptr
    int64_t gmax_ld;
};

int step_smem_bytes();
int step_max_blocks(bool fp8);
// Launches the indexer kernel (when p.phases has kPhaseIndex) and then the
// cooperative kernel for the remaining phases; mid_event (or nullptr) is recorded
// on the stream between the two.
cudaError_t launch_step(const CUtensorMap* kmap, const StepParams& p, bool fp8, cudaStream_t s,
                        cudaEvent_t mid_event = nullptr);

}  // namespace dsa
