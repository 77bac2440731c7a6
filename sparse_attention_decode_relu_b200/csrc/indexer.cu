// indexer.cu -- stage 1 of the DSA decode/verify step: the ReLU indexer scan.
//
//   I[t,s] = scale[s] * sum_{j<16} w[t,j] * ReLU(q_idx[t,j,:] . k_idx[s,:])
//
// NaiveAI research page (naive.ai/en/research), "Technical Details > Model
// Architecture": the lightweight indexer scores the full history, so this is
// the one stage whose cost grows with the context; "Hybrid SWA-DSA
// Architecture": 16 indexer query heads.  The scoring form is the DSA
// indexer's (the page names it but prints no formula).
//
// Design (sm_100a): a persistent grid streams the key cache once.  Tiles of 128
// keys arrive by TMA (cp.async.bulk.tensor) into a 4-stage shared-memory ring
// completed on mbarriers; bf16 keys land 128B-swizzled so the warp MMA operand
// loads are bank-conflict free, FP8-E4M3 keys are widened exactly to bf16 in
// shared memory first.  The indexer queries and head weights arrive once by
// bulk copy.  Each warp owns one query (or a share of one when T < 8) and keeps
// its 16 heads x 64 dims in registers as the N side of m16n8k16 tensor-core
// products whose M side is 16 keys at a time.  The epilogue applies ReLU and
// the head weights, reduces the 16 heads in a fixed order (two quad shuffles),
// and writes fp32 scores.  Positions beyond a query's pos[t] get -inf.
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kStages = 4;
constexpr int kThreads = 256;   // 8 warps; a 128-key tile is 8 blocks of 16 keys

template <bool FP8>
struct IndexerSmem {
    static constexpr int raw_bytes = kKeyTile * kDI * (FP8 ? 1 : 2);
    static constexpr int cvt_bytes = FP8 ? kKeyTile * kDI * 2 : 0;
    static constexpr int q_bytes = kMaxT * kHI * kDI * 2;
    static constexpr int scale_bytes = kKeyTile * 4;
    static constexpr int bytes = 1024 /*align slack*/ + kStages * raw_bytes + cvt_bytes + q_bytes + kMaxT * kHI * 4 +
                                 kStages * scale_bytes + (kStages + 1) * 8;
};

// Warps per query: 8 / T rounded to a power of two, so every query gets the
// same share of the tile.  A warp keeps its query's 16 x 64 indexer heads in
// registers and walks its share of the tile's 16-key blocks.
template <int T>
struct WarpMap {
    static constexpr int TP = T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : 8;
    static constexpr int kWpq = 8 / TP;        // warps per query
    static constexpr int kBlocks = 8 / kWpq;   // 16-key blocks per warp per tile
};

template <int T, bool FP8>
__global__ void __launch_bounds__(kThreads, 2)
    indexer_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap smap,
                   const IndexerParams p)
{
    using S = IndexerSmem<FP8>;
    using M = WarpMap<T>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;                                            // kStages x raw tile
    uint8_t* cvt = ring + kStages * S::raw_bytes;                    // FP8: widened bf16 tile (swizzled)
    uint16_t* q_s = reinterpret_cast<uint16_t*>(cvt + S::cvt_bytes); // [T][16][64] bf16
    float* w_s = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(q_s) + S::q_bytes);
    float* sc_s = w_s + kMaxT * kHI;                                 // kStages x 128 per-token scales
    uint64_t* full = reinterpret_cast<uint64_t*>(sc_s + kStages * kKeyTile);
    uint64_t* setup = full + kStages;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int ntiles = (p.n_max + kKeyTile - 1) / kKeyTile;
    const bool scaled = p.scale != nullptr;
    const uint32_t tile_tx = S::raw_bytes + (scaled ? S::scale_bytes : 0);
    // One tile: 128 key rows, plus their per-token scales when there are any.
    auto load_tile = [&](int stage, int tile) {
        mbar_arrive_expect_tx(&full[stage], tile_tx);
        tma_load_2d(ring + stage * S::raw_bytes, &kmap, 0, tile * kKeyTile, &full[stage]);
        if (scaled) tma_load_1d(sc_s + stage * kKeyTile, &smap, tile * kKeyTile, &full[stage]);
    };

    int issued = 0;   // tiles issued by thread 0
    if (tid == 0) {
        prefetch_tmap(&kmap);
        if (scaled) prefetch_tmap(&smap);
        for (int s = 0; s < kStages + 1; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(setup, T * kHI * kDI * 2 + T * kHI * 4);
        bulk_g2s(q_s, p.q_idx, T * kHI * kDI * 2, setup);
        bulk_g2s(w_s, p.w, T * kHI * 4, setup);
        for (int s = 0; s < kStages; ++s) {
            const int tile = blockIdx.x + s * gridDim.x;
            if (tile >= ntiles) break;
            load_tile(s, tile);
            ++issued;
        }
    }
    if (p.zero != nullptr)   // clear the next stage's counters (nothing reads them before this grid ends)
        for (int i = blockIdx.x * kThreads + tid; i < p.zero_words; i += gridDim.x * kThreads) p.zero[i] = 0u;
    __syncthreads();
    bool ok = mbar_wait(setup, 0, p.err);

    const int t = warp / M::kWpq;           // this warp's query
    const bool active = t < T;
    const int kb0 = warp % M::kWpq;
    int pos_t = -1;
#pragma unroll
    for (int i = 0; i < T; ++i)
        if (i == t) pos_t = p.pos[i];
    // B fragments: B[k = dim][n = head]; n-tile nt = heads 8nt..8nt+7.  ldmatrix
    // rows are heads (128 B apart), matrices are consecutive 8-dim slices.
    uint32_t qb[2][4][2];
    float w0 = 0.f, w1 = 0.f, w8 = 0.f, w9 = 0.f;
    uint32_t klo = 0xFFFFFFFFu, khi = 0u;   // key range of the visible scores this lane wrote
    if (active && ok) {
        const uint32_t qbase = smem_u32(q_s + t * kHI * kDI);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int kp = 0; kp < 2; ++kp) {
                const uint32_t a = qbase + (nt * 8 + (lane & 7)) * (kDI * 2) + (kp * 32 + (lane >> 3) * 8) * 2;
                ldsm_x4(a, qb[nt][2 * kp][0], qb[nt][2 * kp][1], qb[nt][2 * kp + 1][0], qb[nt][2 * kp + 1][1]);
            }
        w0 = w_s[t * kHI + 2 * c];
        w1 = w_s[t * kHI + 2 * c + 1];
        w8 = w_s[t * kHI + 8 + 2 * c];
        w9 = w_s[t * kHI + 9 + 2 * c];
    }

    int it = 0;
    bool aborted = __syncthreads_or(!ok);
    for (int tile = blockIdx.x; !aborted && tile < ntiles; tile += gridDim.x, ++it) {
        const int stage = it % kStages;
        ok = mbar_wait(&full[stage], (it / kStages) & 1, p.err);
        if (__syncthreads_or(!ok)) {
            aborted = true;
            break;
        }
        const uint8_t* ktile = ring + stage * S::raw_bytes;
        if constexpr (FP8) {
            // Widen 128 x 64 E4M3 codes to bf16 in the 128B-swizzled layout.
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int chunk = tid + r * kThreads;   // 16-byte piece of the raw tile
                const int row = chunk >> 2, piece = chunk & 3;
                const uint4 v = *reinterpret_cast<const uint4*>(ktile + row * 64 + piece * 16);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    o[2 * i] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w4[i] & 0xFFFFu));
                    o[2 * i + 1] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w4[i] >> 16));
                }
                const int c0 = (2 * piece) ^ (row & 7), c1 = (2 * piece + 1) ^ (row & 7);
                *reinterpret_cast<uint4*>(cvt + row * 128 + c0 * 16) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4*>(cvt + row * 128 + c1 * 16) = make_uint4(o[4], o[5], o[6], o[7]);
            }
            __syncthreads();
            ktile = cvt;
        }

        if (active) {
#pragma unroll 2
            for (int j = 0; j < M::kBlocks; ++j) {
                const int kb = kb0 + M::kWpq * j;
                // Keys kb*16 .. kb*16+15 as A fragments (16 keys x 64 dims), 128B-swizzled rows.
                uint32_t a[4][4];
                const int row = kb * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const uint32_t base = smem_u32(ktile) + row * 128;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int chunk = 2 * kk + (lane >> 4);
                    ldsm_x4(base + ((chunk ^ (row & 7)) << 4), a[kk][0], a[kk][1], a[kk][2], a[kk][3]);
                }
                float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    mma_bf16_16816(acc0, a[kk], qb[0][kk][0], qb[0][kk][1]);
                    mma_bf16_16816(acc1, a[kk], qb[1][kk][0], qb[1][kk][1]);
                }
                // ReLU, head weights, then the 16 heads summed in a fixed order.
                float pa = fmaxf(acc0[0], 0.f) * w0;
                pa = fmaf(fmaxf(acc0[1], 0.f), w1, pa);
                pa = fmaf(fmaxf(acc1[0], 0.f), w8, pa);
                pa = fmaf(fmaxf(acc1[1], 0.f), w9, pa);
                float pb = fmaxf(acc0[2], 0.f) * w0;
                pb = fmaf(fmaxf(acc0[3], 0.f), w1, pb);
                pb = fmaf(fmaxf(acc1[2], 0.f), w8, pb);
                pb = fmaf(fmaxf(acc1[3], 0.f), w9, pb);
                pa += __shfl_xor_sync(0xffffffffu, pa, 1);
                pb += __shfl_xor_sync(0xffffffffu, pb, 1);
                pa += __shfl_xor_sync(0xffffffffu, pa, 2);
                pb += __shfl_xor_sync(0xffffffffu, pb, 2);
                const int s = tile * kKeyTile + kb * 16 + g + 8 * (c & 1);   // lanes c = 0, 1 write
                if (c < 2 && s < p.L) {
                    const float scale = scaled ? sc_s[stage * kKeyTile + kb * 16 + g + 8 * (c & 1)] : 1.0f;
                    const float v = (c == 0 ? pa : pb) * scale;
                    if (s <= pos_t) {
                        p.scores[(int64_t)t * p.ld + s] = v;
                        const uint32_t k = score_key(v);
                        klo = min(klo, k);
                        khi = max(khi, k);
                    } else {
                        p.scores[(int64_t)t * p.ld + s] = -INFINITY;
                    }
                }
            }
        }

        __syncthreads();   // every warp is done with this stage (and with cvt)
        if (tid == 0) {
            const int next = tile + kStages * gridDim.x;
            if (next < ntiles) {
                load_tile(stage, next);
                ++issued;
            }
        }
    }

    griddep_launch_dependents();
    if (aborted) {
        // Let copies still in flight land before the block's shared memory goes away.
        if (tid == 0) {
            mbar_wait(setup, 0, p.err);
            for (int k = it; k < issued; ++k) mbar_wait(&full[k % kStages], (k / kStages) & 1, p.err);
        }
        __syncthreads();
        return;
    }

    // Per-block key range of each query's visible scores, for the top-k stage.
    if (p.mm != nullptr) {
        __shared__ uint32_t wr[2][8];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            klo = min(klo, __shfl_xor_sync(0xffffffffu, klo, o));
            khi = max(khi, __shfl_xor_sync(0xffffffffu, khi, o));
        }
        if (lane == 0) {
            wr[0][warp] = klo;
            wr[1][warp] = khi;
        }
        __syncthreads();
        if (tid < T) {
            uint32_t lo = 0xFFFFFFFFu, hi = 0u;
            for (int w = tid * M::kWpq; w < (tid + 1) * M::kWpq; ++w) {
                lo = min(lo, wr[0][w]);
                hi = max(hi, wr[1][w]);
            }
            reinterpret_cast<uint2*>(p.mm)[(int64_t)blockIdx.x * kMaxT + tid] = make_uint2(lo, hi);
        }
    }

    // Positions no query can see (s >= n_max): -inf, as the stage's contract states.
    const int64_t tail0 = (int64_t)ntiles * kKeyTile;
    for (int64_t s = tail0 + (int64_t)blockIdx.x * kThreads + tid; s < p.L; s += (int64_t)gridDim.x * kThreads)
#pragma unroll
        for (int tt = 0; tt < T; ++tt) p.scores[(int64_t)tt * p.ld + s] = -INFINITY;
}

template <int T, bool FP8>
cudaError_t launch_t(const CUtensorMap* kmap, const CUtensorMap* smap, const IndexerParams& p, int grid,
                     cudaStream_t s)
{
    constexpr int smem = IndexerSmem<FP8>::bytes;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(indexer_kernel<T, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    indexer_kernel<T, FP8><<<grid, kThreads, smem, s>>>(*kmap, *smap, p);
    return cudaGetLastError();
}

template <int T, bool FP8>
int occupancy_t()
{
    constexpr int smem = IndexerSmem<FP8>::bytes;
    static int cached[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
    cudaFuncSetAttribute(indexer_kernel<T, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, indexer_kernel<T, FP8>, kThreads, smem) != cudaSuccess || n < 1)
        n = 1;
    if (dev >= 0 && dev < 64) cached[dev] = n;
    return n;
}

}  // namespace

#define DSA_INDEXER_DISPATCH(FN, ...)                                              \
    switch (T) {                                                                   \
    case 1: return fp8 ? FN<1, true>(__VA_ARGS__) : FN<1, false>(__VA_ARGS__);     \
    case 2: return fp8 ? FN<2, true>(__VA_ARGS__) : FN<2, false>(__VA_ARGS__);     \
    case 3: return fp8 ? FN<3, true>(__VA_ARGS__) : FN<3, false>(__VA_ARGS__);     \
    case 4: return fp8 ? FN<4, true>(__VA_ARGS__) : FN<4, false>(__VA_ARGS__);     \
    case 5: return fp8 ? FN<5, true>(__VA_ARGS__) : FN<5, false>(__VA_ARGS__);     \
    case 6: return fp8 ? FN<6, true>(__VA_ARGS__) : FN<6, false>(__VA_ARGS__);     \
    case 7: return fp8 ? FN<7, true>(__VA_ARGS__) : FN<7, false>(__VA_ARGS__);     \
    default: return fp8 ? FN<8, true>(__VA_ARGS__) : FN<8, false>(__VA_ARGS__);    \
    }

cudaError_t launch_indexer(const CUtensorMap* kmap, const CUtensorMap* smap, const IndexerParams& p, int T, bool fp8,
                           int grid, cudaStream_t s)
{
    DSA_INDEXER_DISPATCH(launch_t, kmap, smap, p, grid, s)
}

int indexer_max_ctas_per_sm(int T, bool fp8)
{
    DSA_INDEXER_DISPATCH(occupancy_t)
}

}  // namespace dsa
