// attention.cu -- stage 3 of the DSA decode/verify step: softmax attention of the
// 64 query heads over only the selected K/V rows (GQA, 4 KV groups, head dim 128).
//
// NaiveAI research page (naive.ai/en/research), "Technical Details > Hybrid
// SWA-DSA Architecture": GQA with four KV groups over the top-2,048 selection;
// "NaiveRT > Optimizing inside the kernel": selected K/V rows are staged in
// shared memory by split before computation, and the tensor-core mapping is
// chosen so no head rows are padding.
//
// Design (sm_100a): a query's selected rows are cut into splits; one block of 4
// warps handles one (query, split), warp g owning KV group g and its 16 query
// heads -- exactly the 16 rows of an m16n8k16 tile, so nothing is padded.  Whole
// 2 KiB token rows (K then V of all four groups) are gathered by one bulk async
// copy each (cp.async.bulk, completing on an mbarrier) into a 3-stage ring of
// 16-row tiles with a 2064-byte pitch, which keeps the ldmatrix row addresses on
// distinct banks.  Scores and P.V run on tensor cores with an online softmax in
// fp32 (exp2 domain).  The blocks of one query form a thread-block cluster and
// merge their (max, sum, unnormalised output) partials through distributed
// shared memory in a fixed rank order, so the result does not depend on
// scheduling and no partial state goes through global memory.
#include <cooperative_groups.h>

#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

namespace cg = cooperative_groups;

constexpr int kConsumers = 4;                    // warp g computes KV group g
constexpr int kThreads = (kConsumers + 1) * 32;    // plus one producer warp
constexpr int kTileRows = 16;
constexpr int kStages = 3;
constexpr int kRowBytes = 2048;
constexpr int kPitch = 2064;
constexpr int kMaxRowsPerSplit = 256;
constexpr int kRingBytes = kStages * kTileRows * kPitch;
constexpr int kSmemBytes = kRingBytes + 2 * kStages * 8 + kStages * kTileRows * 4 + kMaxRowsPerSplit * 4 + 16;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxCluster = 16;
static_assert(kH * kD * 4 + kH * 8 <= kRingBytes, "merge buffers reuse the ring");

// grid (C, T) with clusters of C blocks along x: the C blocks of a cluster split
// query t's selected rows.  Warp 4 of a block gathers rows into a 3-stage ring
// (full/empty mbarriers); warp g < 4 owns KV group g (query heads 16g..16g+15).
// The cluster merges its partial softmax states through distributed shared
// memory: block r finalises heads [r*64/C, (r+1)*64/C).
__global__ void __launch_bounds__(kThreads, 1) attn_cluster_kernel(const AttnParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRingBytes);
    uint64_t* empty = full + kStages;
    int32_t* rowidx = reinterpret_cast<int32_t*>(empty + kStages);   // [kStages][16]
    int32_t* sel_s = rowidx + kStages * kTileRows;                    // this block's selected rows
    cg::cluster_group cluster = cg::this_cluster();

    const int split = blockIdx.x, t = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, c = lane & 3;
    const int grp = warp;
    int pos_t = 0;
#pragma unroll
    for (int i = 0; i < kMaxT; ++i)
        if (i == t) pos_t = p.pos[i];
    const int rows_t = min(p.rows, pos_t + 1);
    const int r0 = split * p.rows_per_split;
    const int r1 = min(r0 + p.rows_per_split, rows_t);
    const int ntile = r1 > r0 ? (r1 - r0 + kTileRows - 1) / kTileRows : 0;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumers);
        }
        fence_mbar_init();
    }
    __syncthreads();
    griddep_wait();   // the selection comes from the preceding grid

    bool failed = false;
    float oacc[16][4];
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;

    if (warp == kConsumers) {
        // ---------------- producer: validate the selected rows, gather them whole
        const int32_t* selrow = p.sel + (int64_t)t * p.sel_ld + r0;
        for (int j = lane; j < r1 - r0; j += 32) sel_s[j] = __ldg(selrow + j);
        __syncwarp();
        for (int k = 0; k < ntile && !failed; ++k) {
            const int stage = k % kStages;
            if (k >= kStages && !mbar_wait(&empty[stage], ((k / kStages) - 1) & 1, p.err)) {
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
                const int i = __ffs(none) - 1;
                none &= none - 1;
                uint4* v = reinterpret_cast<uint4*>(dst + i * kPitch + kRowBytes / 2);
                v[lane] = make_uint4(0u, 0u, 0u, 0u);
                v[lane + 32] = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&full[stage], __popc(vmask) * kRowBytes);
            __syncwarp();
            if (valid) bulk_g2s(dst + lane * kPitch, p.kv + (int64_t)s * p.kv_ld, kRowBytes, &full[stage]);
        }
    } else {
        // ---------------- consumers
        // Query heads 16*grp .. 16*grp+15 of token t as A fragments (16 x 128).
        uint32_t qa[8][4];
        {
            const uint16_t* qb = p.q + ((int64_t)t * kH + grp * 16) * kD;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                qa[kk][0] = __ldg(reinterpret_cast<const uint32_t*>(qb + gq * kD + kk * 16 + 2 * c));
                qa[kk][1] = __ldg(reinterpret_cast<const uint32_t*>(qb + (gq + 8) * kD + kk * 16 + 2 * c));
                qa[kk][2] = __ldg(reinterpret_cast<const uint32_t*>(qb + gq * kD + kk * 16 + 8 + 2 * c));
                qa[kk][3] = __ldg(reinterpret_cast<const uint32_t*>(qb + (gq + 8) * kD + kk * 16 + 8 + 2 * c));
            }
        }
        const float sm_scale = kLog2e * rsqrtf(static_cast<float>(kD));
        for (int k = 0; k < ntile; ++k) {
            const int stage = k % kStages;
            if (!mbar_wait(&full[stage], (k / kStages) & 1, p.err)) {
                failed = true;
                break;
            }
            const uint32_t base = smem_u32(ring + stage * kTileRows * kPitch);
            const int32_t* ridx = rowidx + stage * kTileRows;

            // S = Q K^T for 16 keys (two n-tiles of 8).
            float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int kk2 = 0; kk2 < 4; ++kk2) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int key = nt * 8 + (lane & 7);
                    const int dim = kk2 * 32 + (lane >> 3) * 8;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(base + key * kPitch + grp * 256 + dim * 2, b0, b1, b2, b3);
                    mma_bf16_16816(sacc[nt], qa[2 * kk2], b0, b1);
                    mma_bf16_16816(sacc[nt], qa[2 * kk2 + 1], b2, b3);
                }
            }
            // Scale into the exp2 domain and mask rows that were not loaded.
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int key = nt * 8 + 2 * c + (i & 1);
                    sacc[nt][i] = ridx[key] >= 0 ? sacc[nt][i] * sm_scale : -INFINITY;
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
            for (int i = 0; i < 16; ++i) {
                oacc[i][0] *= alpha0;
                oacc[i][1] *= alpha0;
                oacc[i][2] *= alpha1;
                oacc[i][3] *= alpha1;
            }
            uint32_t pa[4];
            pa[0] = pack_bf16(pr[0][0], pr[0][1]);
            pa[1] = pack_bf16(pr[0][2], pr[0][3]);
            pa[2] = pack_bf16(pr[1][0], pr[1][1]);
            pa[3] = pack_bf16(pr[1][2], pr[1][3]);
            // O += P V over 128 dims (16 n-tiles of 8; ldmatrix.trans covers two).
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
            if (lane == 0) mbar_arrive(&empty[stage]);   // this warp is done with the stage
        }
    }

    if (__syncthreads_or(failed)) {
        // A bounded wait ran out: let the copies still in flight land, then
        // contribute an empty partial (every block must reach the cluster barriers).
        if (tid == kConsumers * 32) {
            for (int k = max(0, ntile - kStages); k < ntile; ++k)
                mbar_wait(&full[k % kStages], (k / kStages) & 1, p.err);
        }
        __syncthreads();
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    }

    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    // This block's partial state into its own shared memory (the ring is idle now).
    float* o_s = reinterpret_cast<float*>(ring);                       // [64][128]
    float2* ml_s = reinterpret_cast<float2*>(ring + kH * kD * 4);       // [64]
    if (warp < kConsumers) {
        const int h0 = grp * 16 + gq, h1 = h0 + 8;
        if (c == 0) {
            ml_s[h0] = make_float2(m0, l0);
            ml_s[h1] = make_float2(m1, l1);
        }
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
            *reinterpret_cast<float2*>(o_s + h0 * kD + nd * 8 + 2 * c) = make_float2(oacc[nd][0], oacc[nd][1]);
            *reinterpret_cast<float2*>(o_s + h1 * kD + nd * 8 + 2 * c) = make_float2(oacc[nd][2], oacc[nd][3]);
        }
    }
    cluster.sync();

    // Block `split` merges heads [split*hpc, (split+1)*hpc) over the cluster, in rank
    // order; all remote reads of a step are issued before any is used.
    const int C = p.nsplit;
    const int hpc = kH / C;
    for (int item = tid; warp < kConsumers && item < hpc * (kD / 4); item += kConsumers * 32) {
        const int h = split * hpc + item / (kD / 4);
        const int d4 = item % (kD / 4);
        float2 ml[kMaxCluster];
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r)
            ml[r] = r < C ? cluster.map_shared_rank(ml_s, r)[h] : make_float2(-INFINITY, 0.f);
        float4 o[kMaxCluster];
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r)
            o[r] = r < C ? reinterpret_cast<const float4*>(cluster.map_shared_rank(o_s, r) + h * kD)[d4]
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) M = fmaxf(M, ml[r].x);
        float sink = -INFINITY;
        if (p.sink != nullptr) {
            sink = p.sink[h] * kLog2e;
            M = fmaxf(M, sink);
        }
        float den = (p.sink != nullptr && M != -INFINITY) ? exp2f(sink - M) : 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) {
            if (ml[r].x == -INFINITY) continue;   // an empty split (also every r >= C)
            const float w = exp2f(ml[r].x - M);
            den += w * ml[r].y;
            acc.x += w * o[r].x;
            acc.y += w * o[r].y;
            acc.z += w * o[r].z;
            acc.w += w * o[r].w;
        }
        const float inv = den > 0.f ? 1.0f / den : 0.f;
        uint2 packed;
        packed.x = pack_bf16(acc.x * inv, acc.y * inv);
        packed.y = pack_bf16(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2*>(p.out + ((int64_t)t * kH + h) * kD + d4 * 4) = packed;
    }
    cluster.sync();   // no block leaves while its shared memory may still be read
}

int g_cluster[64][kMaxT + 1] = {};   // chosen cluster size per (device, T); 0 = not yet chosen

}  // namespace

// Blocks per query: the largest of 16, 8, 4 for which all T clusters fit on the
// device at once (one wave); 8 if none does.
int attention_cluster_size(int T)
{
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || T < 1 || T > kMaxT) return 8;
    if (g_cluster[dev][T]) return g_cluster[dev][T];
    cudaFuncSetAttribute(attn_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    cudaFuncSetAttribute(attn_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    int chosen = 8;
    for (int C : {16, 8, 4}) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(C, T, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, attn_cluster_kernel, &cfg) == cudaSuccess && n >= T) {
            chosen = C;
            break;
        }
    }
    cudaGetLastError();
    g_cluster[dev][T] = chosen;
    return chosen;
}

cudaError_t launch_attention(const AttnParams& p, int T, cudaStream_t s)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.nsplit, T, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.nsplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, attn_cluster_kernel, p);
}

}  // namespace dsa
