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
// shared memory first.  Each warp owns 16 keys of a tile: keys are the M side of
// m16n8k16 tensor-core products, the T x 16 indexer query heads are the N side
// and stay in registers for the whole scan.  The epilogue applies ReLU and the
// head weights, reduces the 16 heads in a fixed order (two quad shuffles), and
// writes fp32 scores.  Positions beyond a query's pos[t] get -inf.
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kStages = 4;
constexpr int kThreads = 256;   // 8 warps x 16 keys = one 128-key tile

template <bool FP8>
struct IndexerSmem {
    static constexpr int raw_bytes = kKeyTile * kDI * (FP8 ? 1 : 2);
    static constexpr int cvt_bytes = FP8 ? kKeyTile * kDI * 2 : 0;
    static constexpr int bytes = 1024 /*align slack*/ + kStages * raw_bytes + cvt_bytes + kStages * 8 + kMaxT * kHI * 4;
};

template <int T, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap kmap, const IndexerParams p)
{
    using S = IndexerSmem<FP8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;                                            // kStages x raw tile
    uint8_t* cvt = smem + kStages * S::raw_bytes;                    // FP8: widened bf16 tile (swizzled)
    uint64_t* full = reinterpret_cast<uint64_t*>(cvt + S::cvt_bytes);
    float* w_s = reinterpret_cast<float*>(full + kStages);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int ntiles = (p.n_max + kKeyTile - 1) / kKeyTile;

    if (tid == 0) {
        prefetch_tmap(&kmap);
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    if (tid < T * kHI) w_s[tid] = p.w[tid];
    __syncthreads();

    // Indexer queries as B fragments: B[k = dim][n = head], n-tile nt covers heads 8nt..8nt+7.
    uint32_t qb[T][2][4][2];
#pragma unroll
    for (int t = 0; t < T; ++t)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint16_t* src = p.q_idx + (size_t)(t * kHI + nt * 8 + g) * kDI + kk * 16 + 2 * c;
                qb[t][nt][kk][0] = *reinterpret_cast<const uint32_t*>(src);
                qb[t][nt][kk][1] = *reinterpret_cast<const uint32_t*>(src + 8);
            }

    int issued = 0;   // tiles issued by thread 0
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            const int tile = blockIdx.x + s * gridDim.x;
            if (tile >= ntiles) break;
            mbar_arrive_expect_tx(&full[s], S::raw_bytes);
            tma_load_2d(ring + s * S::raw_bytes, &kmap, 0, tile * kKeyTile, &full[s]);
            ++issued;
        }
    }

    int it = 0;
    bool aborted = false;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        const int stage = it % kStages;
        const uint32_t parity = (it / kStages) & 1;
        const bool ok = mbar_wait(&full[stage], parity, p.err);
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

        // Keys of this warp as A fragments (16 keys x 64 dims), 128B-swizzled rows.
        uint32_t a[4][4];
        {
            const int row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const uint32_t base = smem_u32(ktile) + row * 128;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const int chunk = 2 * kk + (lane >> 4);
                ldsm_x4(base + ((chunk ^ (row & 7)) << 4), a[kk][0], a[kk][1], a[kk][2], a[kk][3]);
            }
        }
        const int s_base = tile * kKeyTile + warp * 16;
        const int s_mine = s_base + g + 8 * (c & 1);   // the key this lane writes (lanes c = 0, 1)
        float scale = 1.0f;
        if (p.scale != nullptr && c < 2 && s_mine < p.L) scale = p.scale[s_mine];

#pragma unroll
        for (int t = 0; t < T; ++t) {
            float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16_16816(acc0, a[kk], qb[t][0][kk][0], qb[t][0][kk][1]);
                mma_bf16_16816(acc1, a[kk], qb[t][1][kk][0], qb[t][1][kk][1]);
            }
            const float w0 = w_s[t * kHI + 2 * c], w1 = w_s[t * kHI + 2 * c + 1];
            const float w8 = w_s[t * kHI + 8 + 2 * c], w9 = w_s[t * kHI + 9 + 2 * c];
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
            if (c < 2 && s_mine < p.L) {
                const float v = (c == 0 ? pa : pb) * scale;
                p.scores[(int64_t)t * p.ld + s_mine] = (s_mine <= p.pos[t]) ? v : -INFINITY;
            }
        }

        __syncthreads();   // every warp is done with this stage (and with cvt)
        if (tid == 0) {
            const int next = tile + kStages * gridDim.x;
            if (next < ntiles) {
                mbar_arrive_expect_tx(&full[stage], S::raw_bytes);
                tma_load_2d(ring + stage * S::raw_bytes, &kmap, 0, next * kKeyTile, &full[stage]);
                ++issued;
            }
        }
    }

    if (aborted) {
        // Let copies still in flight land before the block's shared memory goes away.
        if (tid == 0) {
            for (int k = it; k < issued; ++k) mbar_wait(&full[k % kStages], (k / kStages) & 1, p.err);
        }
        __syncthreads();
        return;
    }

    // Positions no query can see (s >= n_max): -inf, as the stage's contract states.
    const int64_t tail0 = (int64_t)ntiles * kKeyTile;
    for (int64_t s = tail0 + (int64_t)blockIdx.x * kThreads + tid; s < p.L; s += (int64_t)gridDim.x * kThreads)
#pragma unroll
        for (int t = 0; t < T; ++t) p.scores[(int64_t)t * p.ld + s] = -INFINITY;
}

template <int T, bool FP8>
cudaError_t launch_t(const CUtensorMap* kmap, const IndexerParams& p, int grid, cudaStream_t s)
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
    indexer_kernel<T, FP8><<<grid, kThreads, smem, s>>>(*kmap, p);
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

cudaError_t launch_indexer(const CUtensorMap* kmap, const IndexerParams& p, int T, bool fp8, int grid,
                           cudaStream_t s)
{
    DSA_INDEXER_DISPATCH(launch_t, kmap, p, grid, s)
}

int indexer_max_ctas_per_sm(int T, bool fp8)
{
    DSA_INDEXER_DISPATCH(occupancy_t)
}

}  // namespace dsa
