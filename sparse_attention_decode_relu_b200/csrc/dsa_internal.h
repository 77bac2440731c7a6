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
constexpr int kHistBins = 4096;            // first-level radix bins (top 12 key bits)

constexpr int kMaxRowsPerSplit = 256;       // selected rows one attention work item gathers
constexpr int kMaxChunksStep = 1024;        // top-k chunks per query (<= grid)
constexpr int kMaxGrid = 1024;              // blocks of the step kernel
constexpr int kMaxAttnItems = 512;          // (query, split) attention work items
constexpr int kTraceSlots = 32;             // phase-boundary stamps per block
constexpr int kBarCtrlBytes = 128;          // grid barrier arrival counter (its own line)
constexpr int kWsCtrlBytes = kBarCtrlBytes + 128;  // + the exit counter: workspace bytes [0, 256)

// Phases of the step kernel.
enum : int {
    kPhaseIndex = 1,    // indexer scan (scores + per-block key ranges)
    kPhaseRanges = 2,   // per-block key ranges of caller-provided scores
    kPhaseTopk = 4,     // histogram, candidates, ordered emission
    kPhaseAttend = 8,   // split attention + merge
    kPhaseSelectPos = 16,   // selection by position: the last `window` visible positions
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
    uint2* mm;               // [grid][kMaxT] per-block (min, max) key of visible scores
    int32_t mm_slots;
    uint32_t* hist;          // [T][kHistBins]
    uint32_t* list_n;        // [kMaxT] candidates per query
    uint2* list;             // [T][list_ld] (key, position) candidates
    int64_t list_ld;         // candidate-list row stride (the workspace's, not the caller's score stride)
    uint32_t* above;         // [T][kMaxChunksStep] keys above the threshold bin, per chunk
    uint32_t* cuts;          // [kMaxT][4]: threshold bin (cut, ctop) and #keys above it, per query
    uint32_t* zero;          // words phase 1 clears (hist, list_n)
    int32_t zero_words;
    int32_t chunk, nchunk;   // top-k work items: nchunk chunks of `chunk` positions per query
    int32_t* sel;            // [T][sel_ld]
    int64_t sel_ld;
    // attention
    const uint16_t* q;       // [T][64][128] bf16
    const uint16_t* kv;      // [L][kv_ld] bf16
    int64_t kv_ld;
    int32_t rows;            // selected rows per query to read (= topk)
    int32_t rows_per_split;  // multiple of 16, <= kMaxRowsPerSplit
    int32_t nsplit;
    const float* sink;       // [64] or nullptr
    int32_t window;          // kPhaseSelectPos: positions selected per query (<= topk)
    float* po;               // [T][nsplit][64][128] partial outputs
    float2* pml;             // [T][nsplit][64] (max in log2 units, sum)
    uint16_t* out;           // [T][64][128] bf16
    // control
    unsigned long long* trace;   // [grid][kTraceSlots] globaltimer stamps at phase boundaries, or nullptr
    uint32_t* bar_ctrl;      // grid barrier arrival counter (zero at launch)
    int64_t barrier_limit;   // SM clocks a grid-barrier wait spins before it gives up
    uint32_t barrier_extra;  // arrivals a grid barrier waits for beyond the grid (0; 1 = a block that never comes)
    uint32_t* err;
};

int step_smem_bytes();
int step_max_blocks(bool fp8);
cudaError_t launch_step(const CUtensorMap* kmap, const CUtensorMap* smap, const StepParams& p, bool fp8,
                        cudaStream_t s);

}  // namespace dsa
