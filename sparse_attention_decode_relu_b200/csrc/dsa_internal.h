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
constexpr int kMaxChunks = 512;            // top-k chunks per query
constexpr int kMaxSplits = 32;             // attention splits per query
constexpr int kMaxSlots = 1024;            // per-block key-range slots

struct IndexerParams {
    const uint16_t* q_idx;   // [T][16][64] bf16
    const float* w;          // [T][16]
    const float* scale;      // [L] or nullptr
    float* scores;           // [T][ld]
    int64_t ld;
    int32_t L;
    int32_t n_max;           // max_t pos[t] + 1: keys at or beyond it are never visible
    int32_t pos[kMaxT];
    uint32_t* zero;          // words the next stage needs zeroed (or nullptr)
    int32_t zero_words;
    uint32_t* mm;            // [gridDim.x][kMaxT] (min, max) key of the block's visible scores, or nullptr
    uint32_t* err;
};

struct TopkParams {
    const float* scores;     // [T][ld]
    int64_t ld;
    int32_t T;
    int32_t topk;
    int32_t chunk;           // elements per chunk (multiple of 2048)
    int32_t nchunks;
    int32_t pos[kMaxT];
    uint32_t* hist;          // [T][kHistBins], zero on entry of the histogram kernel
    uint32_t* tickets;       // [T], zero on entry of the select kernel
    uint32_t* counts;        // [T][kMaxChunks]
    uint2* cand;             // [T][ld]: (key, position) per chunk region
    uint32_t* mm;            // [mm_slots][kMaxT] per-block (min, max) keys
    int32_t mm_slots;
    int32_t* sel;            // [T][sel_ld]
    int64_t sel_ld;
    uint32_t* err;
};

struct AttnParams {
    const uint16_t* q;       // [T][64][128] bf16
    const uint16_t* kv;      // [L][kv_ld] bf16
    int64_t kv_ld;           // elements per token row (>= 1024)
    const int32_t* sel;      // [T][sel_ld]
    int64_t sel_ld;
    int32_t L;
    int32_t rows;            // selected rows per query to read (= topk)
    int32_t rows_per_split;  // multiple of 16
    int32_t nsplit;          // blocks per query = cluster size
    int32_t pos[kMaxT];
    const float* sink;       // [64] or nullptr
    uint16_t* out;           // [T][64][128] bf16
    uint32_t* err;
};

// Launchers return cudaGetLastError() after the launch.  Kernels after the
// first of a step are launched with programmatic stream serialisation: they
// start their prologue early and wait for the preceding grid before reading
// its output.
cudaError_t launch_indexer(const CUtensorMap* kmap, const CUtensorMap* smap, const IndexerParams& p, int T, bool fp8,
                           int grid, cudaStream_t s);
int indexer_max_ctas_per_sm(int T, bool fp8);
cudaError_t launch_topk_cluster(const TopkParams& p, cudaStream_t s);
int64_t topk_cluster_capacity();   // largest n the cluster path holds
cudaError_t launch_topk_minmax(const TopkParams& p, cudaStream_t s);
cudaError_t launch_topk_hist(const TopkParams& p, cudaStream_t s);
cudaError_t launch_topk_select(const TopkParams& p, cudaStream_t s);
cudaError_t launch_attention(const AttnParams& p, int T, cudaStream_t s);
int attention_cluster_size(int T);   // blocks per query (16, 8 or 4)

}  // namespace dsa
