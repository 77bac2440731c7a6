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
// fp32 (exp2 domain); each block writes its (max, sum, unnormalised output)
// partial and a combine kernel merges the splits in a fixed order, so the result
// does not depend on scheduling.
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 128;
constexpr int kTileRows = 16;
constexpr int kStages = 3;
constexpr int kRowBytes = 2048;
constexpr int kPitch = 2064;
constexpr int kSmemBytes = kStages * kTileRows * kPitch + kStages * 8 + kStages * kTileRows * 4 + 16;
constexpr float kLog2e = 1.4426950408889634f;

__global__ void __launch_bounds__(kThreads) attn_split_kernel(const AttnParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kTileRows * kPitch);
    int32_t* rowidx = reinterpret_cast<int32_t*>(full + kStages);   // [kStages][16]

    const int split = blockIdx.x, t = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, c = lane & 3;
    const int grp = warp;
    const int pos_t = p.pos[t];
    const int rows_t = min(p.rows, pos_t + 1);
    const int r0 = split * p.rows_per_split;
    const int r1 = min(r0 + p.rows_per_split, rows_t);
    const int ntile = r1 > r0 ? (r1 - r0 + kTileRows - 1) / kTileRows : 0;
    const int32_t* selrow = p.sel + (int64_t)t * p.sel_ld;
    const int64_t part = (int64_t)t * p.nsplit + split;

    if (ntile == 0) {
        if (tid < kH) p.part_ml[part * kH + tid] = make_float2(-INFINITY, 0.f);
        return;
    }

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }

    // Query heads 16*grp .. 16*grp+15 of token t as A fragments (16 x 128).
    uint32_t qa[8][4];
    {
        const uint16_t* qb = p.q + ((int64_t)t * kH + grp * 16) * kD;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qa[kk][0] = *reinterpret_cast<const uint32_t*>(qb + gq * kD + kk * 16 + 2 * c);
            qa[kk][1] = *reinterpret_cast<const uint32_t*>(qb + (gq + 8) * kD + kk * 16 + 2 * c);
            qa[kk][2] = *reinterpret_cast<const uint32_t*>(qb + gq * kD + kk * 16 + 8 + 2 * c);
            qa[kk][3] = *reinterpret_cast<const uint32_t*>(qb + (gq + 8) * kD + kk * 16 + 8 + 2 * c);
        }
    }
    __syncthreads();

    // Warp 0 gathers tile k: lane i < 16 validates row i and bulk-copies it.
    auto issue = [&](int k) {
        const int stage = k % kStages;
        uint8_t* dst = ring + stage * kTileRows * kPitch;
        int s = -1;
        bool valid = false;
        if (lane < kTileRows) {
            const int j = r0 + k * kTileRows + lane;
            if (j < r1) {
                s = __ldg(selrow + j);
                valid = s >= 0 && s <= pos_t && s < p.L;
                if (s >= 0 && !valid) atomicOr(p.err, ERR_BAD_INDEX);
            }
            rowidx[stage * kTileRows + lane] = valid ? s : -1;
        }
        const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
        // Rows with nothing to load get a zero V half, so P = 0 never meets stale data.
        uint32_t empty = ~vmask & 0xFFFFu;
        while (empty) {
            const int i = __ffs(empty) - 1;
            empty &= empty - 1;
            uint4* v = reinterpret_cast<uint4*>(dst + i * kPitch + kRowBytes / 2);
            v[lane] = make_uint4(0u, 0u, 0u, 0u);
            v[lane + 32] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(&full[stage], __popc(vmask) * kRowBytes);
        __syncwarp();
        if (valid) bulk_g2s(dst + lane * kPitch, p.kv + (int64_t)s * p.kv_ld, kRowBytes, &full[stage]);
    };

    if (warp == 0)
        for (int k = 0; k < kStages && k < ntile; ++k) issue(k);

    float oacc[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    const float sm_scale = kLog2e * rsqrtf(static_cast<float>(kD));

    int k = 0;
    bool aborted = false;
    for (; k < ntile; ++k) {
        const int stage = k % kStages;
        const bool ok = mbar_wait(&full[stage], (k / kStages) & 1, p.err);
        if (__syncthreads_or(!ok)) {
            aborted = true;
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

        __syncthreads();   // the stage is free again
        if (warp == 0 && k + kStages < ntile) issue(k + kStages);
    }

    if (aborted) {
        if (tid == 0)
            for (int j = k; j < min(ntile, k + kStages); ++j) mbar_wait(&full[j % kStages], (j / kStages) & 1, p.err);
        __syncthreads();
        if (tid < kH) p.part_ml[part * kH + tid] = make_float2(-INFINITY, 0.f);
        return;
    }

    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const int h0 = grp * 16 + gq, h1 = h0 + 8;
    if (c == 0) {
        p.part_ml[part * kH + h0] = make_float2(m0, l0);
        p.part_ml[part * kH + h1] = make_float2(m1, l1);
    }
    float* o0 = p.part_o + (part * kH + h0) * kD;
    float* o1 = p.part_o + (part * kH + h1) * kD;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
        *reinterpret_cast<float2*>(o0 + nd * 8 + 2 * c) = make_float2(oacc[nd][0], oacc[nd][1]);
        *reinterpret_cast<float2*>(o1 + nd * 8 + 2 * c) = make_float2(oacc[nd][2], oacc[nd][3]);
    }
}

// Merge the splits of every (query, head) in split order.  grid (T, 8), 256
// threads: warp w of block y owns head 8y + w, lane l owns dims 4l .. 4l+3.
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnParams p)
{
    const int t = blockIdx.x;
    const int h = blockIdx.y * 8 + (threadIdx.x >> 5);
    const int d = (threadIdx.x & 31) * 4;
    const float2* ml = p.part_ml + (int64_t)t * p.nsplit * kH + h;
    float M = -INFINITY;
    for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, __ldcg(ml + (int64_t)s * kH).x);
    float sink = -INFINITY;
    if (p.sink != nullptr) {
        sink = p.sink[h] * kLog2e;
        M = fmaxf(M, sink);
    }
    float den = (p.sink != nullptr && M != -INFINITY) ? exp2f(sink - M) : 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < p.nsplit; ++s) {
        const float2 v = __ldcg(ml + (int64_t)s * kH);
        if (v.x == -INFINITY) continue;
        const float w = exp2f(v.x - M);
        den += w * v.y;
        const float4 o = __ldcg(reinterpret_cast<const float4*>(
            p.part_o + (((int64_t)t * p.nsplit + s) * kH + h) * kD + d));
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
    }
    const float inv = den > 0.f ? 1.0f / den : 0.f;
    uint2 packed;
    packed.x = pack_bf16(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(p.out + ((int64_t)t * kH + h) * kD + d) = packed;
}

}  // namespace

cudaError_t launch_attention(const AttnParams& p, int T, cudaStream_t s)
{
    static int configured[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(attn_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        configured[dev] = 1;
    }
    attn_split_kernel<<<dim3(p.nsplit, T), kThreads, kSmemBytes, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_combine(const AttnParams& p, int T, cudaStream_t s)
{
    attn_combine_kernel<<<dim3(T, kH / 8), 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace dsa
