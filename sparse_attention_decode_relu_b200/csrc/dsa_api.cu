// dsa_api.cu -- the C ABI of libdsa.so (declared in include/dsa_decode.h):
// argument checks, workspace layout, TMA descriptor set-up and launch sequencing
// of the three stages.  No compute happens on the host.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "../../include/dsa_decode.h"
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {

__device__ uint32_t g_err_word;

namespace {

thread_local std::string t_last_error;
thread_local void* t_stage_events[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
thread_local bool t_stage_events_on = false;
thread_local unsigned long long* t_trace = nullptr;
thread_local long long t_fail_barriers = 0;   // > 0: the next launch's grid barriers wait for a block that never comes
std::atomic<uint64_t> g_launches{0};

dsa_status_t fail(dsa_status_t st, const char* fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return st;
}

dsa_status_t cuda_fail(cudaError_t e, const char* what)
{
    return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

struct DeviceInfo {
    int sms = 0;
    uint32_t* err = nullptr;
};

dsa_status_t device_info(DeviceInfo& info)
{
    static DeviceInfo cache[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(DSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
    if (cache[dev].sms == 0) {
        DeviceInfo d;
        e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_err_word);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
        cache[dev] = d;
    }
    info = cache[dev];
    return DSA_OK;
}

void stage_event(int i, cudaStream_t s)
{
    if (t_stage_events_on && t_stage_events[i]) cudaEventRecord(static_cast<cudaEvent_t>(t_stage_events[i]), s);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// ------------------------------------------------------------------ checks
struct Shape {
    int T = 0;
    int64_t L = 0;
    bool fp8 = false;
    int64_t k_ld = 0;    // elements per indexer key row
    int64_t kv_ld = 0;   // elements per cached token row
};

dsa_status_t check_contig(const dsa_tensor_t* x, const char* name, int dtype, int ndim, const int64_t* dims)
{
    if (!x || !x->data) return fail(DSA_ERR_INVALID_ARG, "%s: null", name);
    if (x->dtype != dtype) return fail(DSA_ERR_INVALID_ARG, "%s: dtype %d, expected %d", name, x->dtype, dtype);
    if (x->ndim != ndim) return fail(DSA_ERR_INVALID_ARG, "%s: ndim %d, expected %d", name, x->ndim, ndim);
    int64_t expect = 1;
    for (int i = ndim - 1; i >= 0; --i) {
        if (dims[i] >= 0 && x->shape[i] != dims[i])
            return fail(i == 0 ? DSA_ERR_INVALID_ARG : DSA_ERR_UNSUPPORTED, "%s: shape[%d] = %lld, expected %lld",
                        name, i, (long long)x->shape[i], (long long)dims[i]);
        if (x->stride[i] != expect)
            return fail(DSA_ERR_INVALID_ARG, "%s: must be contiguous (stride[%d] = %lld)", name, i,
                        (long long)x->stride[i]);
        expect *= x->shape[i];
    }
    if (!aligned16(x->data)) return fail(DSA_ERR_INVALID_ARG, "%s: base not 16-byte aligned", name);
    return DSA_OK;
}

dsa_status_t check_T(int64_t T)
{
    if (T < 1 || T > kMaxT) return fail(DSA_ERR_UNSUPPORTED, "T = %lld query tokens (1..%d supported)", (long long)T, kMaxT);
    return DSA_OK;
}

dsa_status_t check_indexer_inputs(const dsa_tensor_t* q_idx, const dsa_tensor_t* w_idx, const dsa_tensor_t* k,
                                  const int32_t* pos, Shape& sh)
{
    if (!q_idx) return fail(DSA_ERR_INVALID_ARG, "q_idx: null");
    sh.T = static_cast<int>(q_idx->shape[0]);
    dsa_status_t st = check_T(q_idx->shape[0]);
    if (st) return st;
    const int64_t qd[3] = {sh.T, kHI, kDI};
    if ((st = check_contig(q_idx, "q_idx", DSA_BF16, 3, qd))) return st;
    const int64_t wd[2] = {sh.T, kHI};
    if ((st = check_contig(w_idx, "w_idx", DSA_F32, 2, wd))) return st;
    if (!k || !k->data) return fail(DSA_ERR_INVALID_ARG, "k_idx_cache: null");
    if (k->dtype != DSA_BF16 && k->dtype != DSA_FP8_E4M3)
        return fail(DSA_ERR_INVALID_ARG, "k_idx_cache: dtype must be bf16 or fp8-e4m3");
    if (k->ndim != 2) return fail(DSA_ERR_INVALID_ARG, "k_idx_cache: ndim must be 2");
    if (k->shape[1] != kDI) return fail(DSA_ERR_UNSUPPORTED, "k_idx_cache: dim %lld (64 supported)", (long long)k->shape[1]);
    sh.L = k->shape[0];
    if (sh.L < 1 || sh.L > INT32_MAX - 4096) return fail(DSA_ERR_INVALID_ARG, "k_idx_cache: L = %lld", (long long)sh.L);
    sh.fp8 = k->dtype == DSA_FP8_E4M3;
    const int64_t es = sh.fp8 ? 1 : 2;
    if (k->stride[1] != 1 || k->stride[0] < kDI || (k->stride[0] * es) % 16)
        return fail(DSA_ERR_INVALID_ARG, "k_idx_cache: row stride must be >= 64 elements and a multiple of 16 bytes");
    if (!aligned16(k->data)) return fail(DSA_ERR_INVALID_ARG, "k_idx_cache: base not 16-byte aligned");
    if (k->scale && !aligned16(k->scale)) return fail(DSA_ERR_INVALID_ARG, "k_idx_cache.scale: not 16-byte aligned");
    sh.k_ld = k->stride[0];
    if (!pos) return fail(DSA_ERR_INVALID_ARG, "pos: null");
    for (int t = 0; t < sh.T; ++t)
        if (pos[t] < 0 || pos[t] >= sh.L)
            return fail(DSA_ERR_INVALID_ARG, "pos[%d] = %d outside [0, L = %lld)", t, pos[t], (long long)sh.L);
    return DSA_OK;
}

dsa_status_t check_kv(const dsa_tensor_t* kv, Shape& sh)
{
    if (!kv || !kv->data) return fail(DSA_ERR_INVALID_ARG, "kv_cache: null");
    if (kv->dtype != DSA_BF16) return fail(DSA_ERR_INVALID_ARG, "kv_cache: dtype must be bf16");
    if (kv->ndim != 4) return fail(DSA_ERR_INVALID_ARG, "kv_cache: ndim must be 4");
    if (kv->shape[1] != 2 || kv->shape[2] != kG || kv->shape[3] != kD)
        return fail(DSA_ERR_UNSUPPORTED, "kv_cache: shape [L][2][4][128] supported");
    if (kv->stride[3] != 1 || kv->stride[2] != kD || kv->stride[1] != kG * kD || kv->stride[0] < 2 * kG * kD ||
        kv->stride[0] % 8)
        return fail(DSA_ERR_INVALID_ARG, "kv_cache: token rows must be [2][4][128] contiguous, stride a multiple of 8");
    if (!aligned16(kv->data)) return fail(DSA_ERR_INVALID_ARG, "kv_cache: base not 16-byte aligned");
    if (sh.L && kv->shape[0] != sh.L)
        return fail(DSA_ERR_INVALID_ARG, "kv_cache: L = %lld but the key cache has %lld", (long long)kv->shape[0],
                    (long long)sh.L);
    sh.L = kv->shape[0];
    sh.kv_ld = kv->stride[0];
    return DSA_OK;
}

dsa_status_t check_topk(int32_t topk)
{
    if (topk < 1 || topk > kMaxTopk) return fail(DSA_ERR_INVALID_ARG, "topk = %d outside [1, %d]", topk, kMaxTopk);
    return DSA_OK;
}

dsa_status_t check_sel(const dsa_tensor_t* sel, int T, int32_t topk)
{
    if (!sel || !sel->data) return fail(DSA_ERR_INVALID_ARG, "sel_idx: null");
    if (sel->dtype != DSA_I32 || sel->ndim != 2) return fail(DSA_ERR_INVALID_ARG, "sel_idx: int32 [T][topk] expected");
    if (sel->shape[0] != T || sel->shape[1] != topk)
        return fail(DSA_ERR_INVALID_ARG, "sel_idx: shape [%lld][%lld], expected [%d][%d]", (long long)sel->shape[0],
                    (long long)sel->shape[1], T, topk);
    if (sel->stride[1] != 1 || sel->stride[0] < topk)
        return fail(DSA_ERR_INVALID_ARG, "sel_idx: rows must be contiguous with stride >= topk");
    if (!aligned16(sel->data)) return fail(DSA_ERR_INVALID_ARG, "sel_idx: base not 16-byte aligned");
    return DSA_OK;
}

// ------------------------------------------------------------------ workspace
// Device workspace of one step: the control region (barrier and per-query
// words, two radix histograms), per-query cuts, per-sub-segment candidate
// counts, candidate lists, fp32 scores with the largest key of each group of 32
// positions, and the attention splits' partial states.
struct Layout {
    int64_t ld = 0;            // score / candidate row stride (elements)
    int64_t gmax_ld = 0;       // group-maximum row stride (32-position groups)
    size_t ctrl = 0, cuts = 0, seg_n = 0, scores = 0, gmax = 0, list = 0, po = 0, pml = 0;
    size_t total = 0;
};

constexpr size_t ru256(size_t x) { return (x + 255) / 256 * 256; }

// with_scores / with_attn: whether the layout carries the score and the
// attention regions (the allocation-free top-k needs neither).
Layout layout(int T, int64_t L, bool with_scores = true, bool with_attn = true)
{
    Layout l;
    l.ld = round_up(L, 64);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += ru256(bytes);
        return at;
    };
    l.ctrl = take(kWsCtrlBytes);
    l.cuts = take(sizeof(uint32_t) * 4 * kMaxT);
    l.seg_n = take(sizeof(uint32_t) * (size_t)kMaxT * kMaxSeg);
    l.list = take(sizeof(uint2) * (size_t)T * l.ld);
    if (with_scores) {
        l.scores = take(sizeof(float) * (size_t)T * l.ld);
        l.gmax_ld = round_up(L, kKeyTile) / 32;   // every group of the indexer's tiles
        l.gmax = take(sizeof(uint32_t) * (size_t)T * l.gmax_ld);
    }
    if (with_attn) {
        l.po = take(sizeof(float) * (size_t)kMaxT * kMaxSplitsQ * kH * kD);
        l.pml = take(sizeof(float2) * (size_t)kMaxT * kMaxSplitsQ * kH);
    }
    l.total = off;
    return l;
}

dsa_status_t check_ws(void* ws, size_t bytes, const Layout& l)
{
    if (!ws) return fail(DSA_ERR_INVALID_ARG, "workspace: null");
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(DSA_ERR_INVALID_ARG, "workspace: not 256-byte aligned");
    if (bytes < l.total)
        return fail(DSA_ERR_INVALID_ARG, "workspace: %zu bytes, %zu needed", bytes, l.total);
    return DSA_OK;
}

template <typename P>
P* at(void* ws, size_t off) { return reinterpret_cast<P*>(static_cast<char*>(ws) + off); }

// ------------------------------------------------------------------ the step kernel
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// TMA descriptor of the indexer key cache: 128-key tiles; bf16 rows land
// 128B-swizzled (the MMA's shared-memory operand layout), E4M3 rows 64B-swizzled
// (conflict-free row reads for the widening).
dsa_status_t encode_key_map(const dsa_tensor_t* k, const Shape& sh, CUtensorMap& map)
{
    auto enc = encode_fn();
    if (!enc) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDI), static_cast<cuuint64_t>(sh.L)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(sh.k_ld * (sh.fp8 ? 1 : 2))};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kDI), static_cast<cuuint32_t>(kKeyTile)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&map, sh.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k->data, dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     sh.fp8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return DSA_OK;
}

int grid_blocks(const DeviceInfo& dev, bool fp8)
{
    static int cache[64][2] = {};
    int d = 0;
    cudaGetDevice(&d);
    if (d >= 0 && d < 64 && cache[d][fp8]) return cache[d][fp8];
    int g = step_max_blocks(fp8);
    if (g > kMaxGrid) g = kMaxGrid;
    if (g < 1) g = dev.sms > 0 ? dev.sms : 1;
    if (d >= 0 && d < 64) cache[d][fp8] = g;
    return g;
}

// Fill the top-k part of the parameters (work split, workspace pointers): one
// extraction item per (query, chunk) and block, chunks a multiple of 256
// positions so that each warp's eighth starts 128-byte aligned.
void topk_params(StepParams& p, void* ws, const Layout& l)
{
    p.cuts = at<uint32_t>(ws, l.cuts);
    p.seg_n = at<uint32_t>(ws, l.seg_n);
    p.list = at<uint2>(ws, l.list);
    p.list_ld = l.ld;
    int nchunk = p.grid / p.T;
    if (nchunk < 1) nchunk = 1;
    if (nchunk > kMaxChunksStep) nchunk = kMaxChunksStep;
    int64_t chunk = round_up((p.n_max + nchunk - 1) / nchunk, 256);
    if (chunk < 256) chunk = 256;
    p.chunk = static_cast<int32_t>(chunk);
    p.nchunk = static_cast<int32_t>((p.n_max + chunk - 1) / chunk);
    if (p.nchunk < 1) p.nchunk = 1;
}

// Attention work split: items (query, row split), about one per block; splits
// of a multiple of 16 rows, at least kMinRowsPerSplit (so at most kMaxSplitsQ
// per query) and at most kMaxRowsPerSplit.
void attn_params(StepParams& p, void* ws, const Layout& l, int32_t rows)
{
    int64_t nsplit = p.grid / p.T;
    const int64_t most = (rows + kMinRowsPerSplit - 1) / kMinRowsPerSplit;
    if (nsplit > most) nsplit = most;
    if (nsplit < 1) nsplit = 1;
    int64_t rps = round_up((rows + nsplit - 1) / nsplit, 16);
    if (rps > kMaxRowsPerSplit) rps = kMaxRowsPerSplit;
    p.rows = rows;
    p.rows_per_split = static_cast<int32_t>(rps);
    p.nsplit = static_cast<int32_t>((rows + rps - 1) / rps);
    p.po = at<float>(ws, l.po);
    p.pml = at<float2>(ws, l.pml);
}

dsa_status_t launch(const CUtensorMap& map, StepParams& p, bool fp8, void* ws, const Layout& l, cudaStream_t stream)
{
    cudaError_t e;
    // Every launch with a workspace uses its control region: zero from the
    // workspace's creation on, and each launch leaves it ready for the next.
    p.ctrl = ws != nullptr ? at<uint32_t>(ws, l.ctrl) : nullptr;
    p.trace = t_trace;
    p.barrier_limit = kWaitLimitCycles;
    p.barrier_extra = 0;
    if (t_fail_barriers > 0 && p.ctrl != nullptr) {   // one launch only
        p.barrier_limit = t_fail_barriers;
        p.barrier_extra = 1;
        t_fail_barriers = 0;
    }
    cudaEvent_t mid = t_stage_events_on ? static_cast<cudaEvent_t>(t_stage_events[1]) : nullptr;
    if ((e = launch_step(&map, p, fp8, stream, mid)) != cudaSuccess) return cuda_fail(e, "step launch");
    g_launches += ((p.phases & kPhaseIndex) != 0) + ((p.phases & ~kPhaseIndex) != 0);   // indexer, cooperative kernel
    return DSA_OK;
}

void set_pos(StepParams& p, const int32_t* pos, int T)
{
    p.T = T;
    int n_max = 0;
    for (int t = 0; t < kMaxT; ++t) {
        p.pos[t] = t < T ? pos[t] : 0;
        if (t < T && pos[t] + 1 > n_max) n_max = pos[t] + 1;
    }
    p.n_max = n_max;
}

dsa_status_t check_decode_args(const dsa_tensor_t* q, const dsa_tensor_t* q_idx, const dsa_tensor_t* w_idx,
                               const dsa_tensor_t* k_idx_cache, const dsa_tensor_t* kv_cache, const int32_t* pos,
                               int32_t topk, dsa_tensor_t* out, dsa_tensor_t* sel_idx, Shape& sh)
{
    dsa_status_t st = check_indexer_inputs(q_idx, w_idx, k_idx_cache, pos, sh);
    if (st) return st;
    const int64_t qd[3] = {sh.T, kH, kD};
    if ((st = check_contig(q, "q", DSA_BF16, 3, qd))) return st;
    if ((st = check_kv(kv_cache, sh))) return st;
    if ((st = check_topk(topk))) return st;
    if ((st = check_contig(out, "out", DSA_BF16, 3, qd))) return st;
    if ((st = check_sel(sel_idx, sh.T, topk))) return st;
    return DSA_OK;
}

// ------------------------------------------------------------------ no-allocation top-k
// Scratch for dsa_topk_from_scores_noalloc: a file-scope device array, so that
// entry point never allocates.  Sized for T <= 8 queries and L <= 262144 scores
// per query: the control region (barrier words, two radix histograms), cuts,
// per-sub-segment counts and the candidate lists (about 17.3 MB per device,
// held until the process exits).  Static device memory starts zeroed, which is
// the state the control region needs before its first use.
constexpr int64_t kNoAllocMaxL = 262144;
constexpr size_t kNoAllocBytes = ru256(kWsCtrlBytes) + ru256(sizeof(uint32_t) * 4 * kMaxT) +
                                 ru256(sizeof(uint32_t) * (size_t)kMaxT * kMaxSeg) +
                                 ru256(sizeof(uint2) * (size_t)kMaxT * ((kNoAllocMaxL + 63) / 64 * 64));

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

// Device address of the scratch array on the current device.  The host-side
// name g_noalloc_scratch is only a stand-in, so the address is looked up once
// per device (with that device current) and cached.
std::atomic<void*> g_noalloc_ptr[64];

dsa_status_t noalloc_scratch(void** ptr)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(DSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
    void* p = g_noalloc_ptr[dev].load();
    if (!p) {
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
        g_noalloc_ptr[dev].store(p);
    }
    *ptr = p;
    return DSA_OK;
}

dsa_status_t run_topk_stage(const float* scores, int32_t T, int64_t L, int64_t ld, const int32_t* pos, int32_t topk,
                            int32_t* sel_idx, int64_t sel_ld, void* ws, const Layout& l, cudaStream_t stream)
{
    DeviceInfo dev;
    dsa_status_t st = device_info(dev);
    if (st) return st;
    StepParams p{};
    p.phases = kPhaseHistScores | kPhaseTopk;
    p.grid = grid_blocks(dev, false);
    set_pos(p, pos, T);
    p.L = static_cast<int32_t>(L);
    p.topk = topk;
    p.scores = const_cast<float*>(scores);
    p.ld = ld;
    p.sel = sel_idx;
    p.sel_ld = sel_ld;
    p.err = dev.err;
    topk_params(p, ws, l);
    CUtensorMap none;
    std::memset(&none, 0, sizeof none);
    return launch(none, p, false, ws, l, stream);
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

size_t dsa_workspace_bytes(int32_t T, int64_t L, int32_t topk)
{
    if (T < 1 || T > kMaxT || L < 1 || L > INT32_MAX - 4096 || topk < 1 || topk > kMaxTopk) return 0;
    return layout(T, L).total;
}

// Short-context bypass: when every query sees at most topk positions the top-k
// selects everything, so the step skips scoring and selects by position.
static std::atomic<int> g_bypass{1};

static dsa_status_t decode_ws(const dsa_tensor_t* q, const dsa_tensor_t* q_idx, const dsa_tensor_t* w_idx,
                       const dsa_tensor_t* k_idx_cache, const dsa_tensor_t* kv_cache, const int32_t* pos, int32_t topk,
                       const float* sink, dsa_tensor_t* out, dsa_tensor_t* sel_idx, dsa_stream_t stream_,
                       void* workspace, size_t workspace_bytes, const int32_t* pos_device = nullptr)
{
    t_last_error.clear();
    Shape sh;
    const int32_t zeros[kMaxT] = {0, 0, 0, 0, 0, 0, 0, 0};   // stand-in host positions for a device pos
    if (pos_device) {
        if (reinterpret_cast<uintptr_t>(pos_device) & 3u) return fail(DSA_ERR_INVALID_ARG, "pos_device: not 4-byte aligned");
        pos = zeros;
    }
    dsa_status_t st = check_decode_args(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk, out, sel_idx, sh);
    if (st) return st;
    if (sink && !aligned16(sink)) return fail(DSA_ERR_INVALID_ARG, "sink: not 16-byte aligned");
    const Layout l = layout(sh.T, sh.L);
    if ((st = check_ws(workspace, workspace_bytes, l))) return st;
    DeviceInfo dev;
    if ((st = device_info(dev))) return st;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    CUtensorMap map;
    if ((st = encode_key_map(k_idx_cache, sh, map))) return st;
    StepParams p{};
    p.phases = kPhaseIndex | kPhaseTopk | kPhaseAttend;
    p.grid = grid_blocks(dev, sh.fp8);
    set_pos(p, pos, sh.T);
    if (pos_device) {   // positions are read at launch: split the work over the whole cache
        p.pos_dev = pos_device;
        p.n_max = static_cast<int32_t>(sh.L);
    } else if (g_bypass.load() && p.n_max <= topk) {
        p.phases = kPhaseSelectPos | kPhaseAttend;
        p.window = topk;
    }
    p.L = static_cast<int32_t>(sh.L);
    p.topk = topk;
    p.q_idx = static_cast<const uint16_t*>(q_idx->data);
    p.w = static_cast<const float*>(w_idx->data);
    p.scale = k_idx_cache->scale;
    p.scores = at<float>(workspace, l.scores);
    p.ld = l.ld;
    p.gmax = at<uint32_t>(workspace, l.gmax);
    p.gmax_ld = l.gmax_ld;
    p.sel = static_cast<int32_t*>(sel_idx->data);
    p.sel_ld = sel_idx->stride[0];
    p.q = static_cast<const uint16_t*>(q->data);
    p.kv = static_cast<const uint16_t*>(kv_cache->data);
    p.kv_ld = sh.kv_ld;
    p.sink = sink;
    p.out = static_cast<uint16_t*>(out->data);
    p.err = dev.err;
    topk_params(p, workspace, l);
    attn_params(p, workspace, l, topk);
    stage_event(0, stream);
    st = launch(map, p, sh.fp8, workspace, l, stream);   // events[1] between the indexer and the cooperative kernel
    for (int i = 2; i < 5; ++i) stage_event(i, stream);
    return st;
}

dsa_status_t dsa_decode_ws(const dsa_tensor_t* q, const dsa_tensor_t* q_idx, const dsa_tensor_t* w_idx,
                           const dsa_tensor_t* k_idx_cache, const dsa_tensor_t* kv_cache, const int32_t* pos,
                           int32_t topk, dsa_tensor_t* out, dsa_tensor_t* sel_idx, dsa_stream_t stream,
                           void* workspace, size_t workspace_bytes)
{
    return decode_ws(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk, nullptr, out, sel_idx, stream, workspace,
                     workspace_bytes);
}

dsa_status_t dsa_decode_sink_ws(const dsa_tensor_t* q, const dsa_tensor_t* q_idx, const dsa_tensor_t* w_idx,
                                const dsa_tensor_t* k_idx_cache, const dsa_tensor_t* kv_cache, const int32_t* pos,
                                int32_t topk, const float* sink, dsa_tensor_t* out, dsa_tensor_t* sel_idx,
                                dsa_stream_t stream, void* workspace, size_t workspace_bytes)
{
    if (!sink) return fail(DSA_ERR_INVALID_ARG, "sink: null");
    return decode_ws(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk, sink, out, sel_idx, stream, workspace,
                     workspace_bytes);
}

void dsa_set_short_context_bypass(int32_t enable) { g_bypass.store(enable != 0 ? 1 : 0); }

dsa_status_t dsa_decode_devpos_ws(const dsa_tensor_t* q, const dsa_tensor_t* q_idx, const dsa_tensor_t* w_idx,
                                  const dsa_tensor_t* k_idx_cache, const dsa_tensor_t* kv_cache,
                                  const int32_t* pos_device, int32_t topk, const float* sink, dsa_tensor_t* out,
                                  dsa_tensor_t* sel_idx, dsa_stream_t stream, void* workspace, size_t workspace_bytes)
{
    if (!pos_device) return fail(DSA_ERR_INVALID_ARG, "pos_device: null");
    return decode_ws(q, q_idx, w_idx, k_idx_cache, kv_cache, nullptr, topk, sink, out, sel_idx, stream, workspace,
                     workspace_bytes, pos_device);
}

dsa_status_t dsa_swa_decode(const dsa_tensor_t* q, const dsa_tensor_t* kv_cache, const int32_t* pos, int32_t window,
                            const float* sink, dsa_tensor_t* out, dsa_stream_t stream_, void* workspace,
                            size_t workspace_bytes)
{
    t_last_error.clear();
    if (!q) return fail(DSA_ERR_INVALID_ARG, "q: null");
    Shape sh;
    sh.T = static_cast<int>(q->shape[0]);
    dsa_status_t st = check_T(q->shape[0]);
    if (st) return st;
    const int64_t qd[3] = {sh.T, kH, kD};
    if ((st = check_contig(q, "q", DSA_BF16, 3, qd))) return st;
    if ((st = check_kv(kv_cache, sh))) return st;
    if (window < 1 || window > kMaxTopk) return fail(DSA_ERR_INVALID_ARG, "window = %d outside [1, %d]", window, kMaxTopk);
    if ((st = check_contig(out, "out", DSA_BF16, 3, qd))) return st;
    if (!pos) return fail(DSA_ERR_INVALID_ARG, "pos: null");
    for (int t = 0; t < sh.T; ++t)
        if (pos[t] < 0 || pos[t] >= sh.L) return fail(DSA_ERR_INVALID_ARG, "pos[%d] = %d outside [0, L)", t, pos[t]);
    if (sink && !aligned16(sink)) return fail(DSA_ERR_INVALID_ARG, "sink: not 16-byte aligned");
    const Layout l = layout(sh.T, sh.L);
    if ((st = check_ws(workspace, workspace_bytes, l))) return st;
    DeviceInfo dev;
    if ((st = device_info(dev))) return st;
    StepParams p{};
    p.phases = kPhaseSelectPos | kPhaseAttend;
    p.grid = grid_blocks(dev, false);
    set_pos(p, pos, sh.T);
    p.L = static_cast<int32_t>(sh.L);
    p.topk = window;
    p.window = window;
    p.sel = at<int32_t>(workspace, l.list);   // the window's positions live in the candidate-list region
    p.sel_ld = window;
    p.q = static_cast<const uint16_t*>(q->data);
    p.kv = static_cast<const uint16_t*>(kv_cache->data);
    p.kv_ld = sh.kv_ld;
    p.sink = sink;
    p.out = static_cast<uint16_t*>(out->data);
    p.err = dev.err;
    attn_params(p, workspace, l, window);
    CUtensorMap none;
    std::memset(&none, 0, sizeof none);
    return launch(none, p, false, workspace, l, reinterpret_cast<cudaStream_t>(stream_));
}

dsa_status_t dsa_decode(const dsa_tensor_t* q, const dsa_tensor_t* q_idx, const dsa_tensor_t* w_idx,
                        const dsa_tensor_t* k_idx_cache, const dsa_tensor_t* kv_cache, const int32_t* pos,
                        int32_t topk, dsa_tensor_t* out, dsa_tensor_t* sel_idx, dsa_stream_t stream_)
{
    t_last_error.clear();
    Shape sh;
    dsa_status_t st = check_decode_args(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk, out, sel_idx, sh);
    if (st) return st;
    const size_t bytes = layout(sh.T, sh.L).total;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    void* ws = nullptr;
    cudaError_t e = cudaMallocAsync(&ws, bytes, stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
    e = cudaMemsetAsync(ws, 0, kWsCtrlBytes, stream);
    if (e != cudaSuccess) {
        cudaFreeAsync(ws, stream);
        return cuda_fail(e, "workspace control reset");
    }
    st = dsa_decode_ws(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk, out, sel_idx, stream_, ws, bytes);
    e = cudaFreeAsync(ws, stream);
    if (st == DSA_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(workspace)");
    return st;
}

dsa_status_t dsa_index_scores(const dsa_tensor_t* q_idx, const dsa_tensor_t* w_idx, const dsa_tensor_t* k_idx_cache,
                              const int32_t* pos, float* scores, int64_t ld, dsa_stream_t stream_)
{
    t_last_error.clear();
    Shape sh;
    dsa_status_t st = check_indexer_inputs(q_idx, w_idx, k_idx_cache, pos, sh);
    if (st) return st;
    if (!scores || !aligned16(scores)) return fail(DSA_ERR_INVALID_ARG, "scores: null or not 16-byte aligned");
    if (ld < sh.L || ld % 4) return fail(DSA_ERR_INVALID_ARG, "scores: ld = %lld must be >= L and a multiple of 4", (long long)ld);
    DeviceInfo dev;
    if ((st = device_info(dev))) return st;
    CUtensorMap map;
    if ((st = encode_key_map(k_idx_cache, sh, map))) return st;
    StepParams p{};
    p.phases = kPhaseIndex;
    p.grid = grid_blocks(dev, sh.fp8);
    set_pos(p, pos, sh.T);
    p.L = static_cast<int32_t>(sh.L);
    p.q_idx = static_cast<const uint16_t*>(q_idx->data);
    p.w = static_cast<const float*>(w_idx->data);
    p.scale = k_idx_cache->scale;
    p.scores = scores;
    p.ld = ld;
    p.err = dev.err;
    const Layout l{};
    return launch(map, p, sh.fp8, nullptr, l, reinterpret_cast<cudaStream_t>(stream_));
}

dsa_status_t dsa_topk_from_scores(const float* scores, int32_t T, int64_t L, int64_t ld, const int32_t* pos,
                                  int32_t topk, int32_t* sel_idx, int64_t sel_ld, dsa_stream_t stream_,
                                  void* workspace, size_t workspace_bytes)
{
    t_last_error.clear();
    dsa_status_t st = check_T(T);
    if (st) return st;
    if ((st = check_topk(topk))) return st;
    if (L < 1 || L > INT32_MAX - 4096) return fail(DSA_ERR_INVALID_ARG, "L = %lld", (long long)L);
    if (!scores || !aligned16(scores)) return fail(DSA_ERR_INVALID_ARG, "scores: null or not 16-byte aligned");
    if (ld < L || ld % 4) return fail(DSA_ERR_INVALID_ARG, "scores: ld must be >= L and a multiple of 4");
    if (!sel_idx || !aligned16(sel_idx) || sel_ld < topk)
        return fail(DSA_ERR_INVALID_ARG, "sel_idx: null, unaligned, or sel_ld < topk");
    if (!pos) return fail(DSA_ERR_INVALID_ARG, "pos: null");
    for (int t = 0; t < T; ++t)
        if (pos[t] < 0 || pos[t] >= L) return fail(DSA_ERR_INVALID_ARG, "pos[%d] = %d outside [0, L)", t, pos[t]);
    const Layout l = layout(T, L);
    if ((st = check_ws(workspace, workspace_bytes, l))) return st;
    return run_topk_stage(scores, T, L, ld, pos, topk, sel_idx, sel_ld, workspace, l,
                          reinterpret_cast<cudaStream_t>(stream_));
}

dsa_status_t dsa_topk_from_scores_noalloc(const float* scores, int32_t T, int64_t L, int64_t ld,
                                          const int32_t* pos, int32_t topk, int32_t* sel_idx, int64_t sel_ld,
                                          dsa_stream_t stream_)
{
    t_last_error.clear();
    dsa_status_t st = check_T(T);
    if (st) return st;
    if ((st = check_topk(topk))) return st;
    if (L < 1) return fail(DSA_ERR_INVALID_ARG, "L = %lld", (long long)L);
    if (L > kNoAllocMaxL)
        return fail(DSA_ERR_INVALID_ARG, "L = %lld exceeds the no-allocation scratch limit of %lld scores per query",
                    (long long)L, (long long)kNoAllocMaxL);
    if (!scores || !aligned16(scores)) return fail(DSA_ERR_INVALID_ARG, "scores: null or not 16-byte aligned");
    if (ld < L || ld % 4) return fail(DSA_ERR_INVALID_ARG, "scores: ld must be >= L and a multiple of 4");
    if (!sel_idx || !aligned16(sel_idx) || sel_ld < topk)
        return fail(DSA_ERR_INVALID_ARG, "sel_idx: null, unaligned, or sel_ld < topk");
    if (!pos) return fail(DSA_ERR_INVALID_ARG, "pos: null");
    for (int t = 0; t < T; ++t)
        if (pos[t] < 0 || pos[t] >= L) return fail(DSA_ERR_INVALID_ARG, "pos[%d] = %d outside [0, L)", t, pos[t]);
    const Layout l = layout(T, L, false, false);
    if (l.total > kNoAllocBytes) return fail(DSA_ERR_INVALID_ARG, "no-allocation scratch too small");
    void* ws = nullptr;
    if ((st = noalloc_scratch(&ws))) return st;
    return run_topk_stage(scores, T, L, ld, pos, topk, sel_idx, sel_ld, ws, l, reinterpret_cast<cudaStream_t>(stream_));
}

dsa_status_t dsa_sparse_attn(const dsa_tensor_t* q, const dsa_tensor_t* kv_cache, const dsa_tensor_t* sel_idx,
                             const int32_t* pos, const float* sink, dsa_tensor_t* out, dsa_stream_t stream_,
                             void* workspace, size_t workspace_bytes)
{
    t_last_error.clear();
    if (!q) return fail(DSA_ERR_INVALID_ARG, "q: null");
    Shape sh;
    sh.T = static_cast<int>(q->shape[0]);
    dsa_status_t st = check_T(q->shape[0]);
    if (st) return st;
    const int64_t qd[3] = {sh.T, kH, kD};
    if ((st = check_contig(q, "q", DSA_BF16, 3, qd))) return st;
    if ((st = check_kv(kv_cache, sh))) return st;
    if (!sel_idx) return fail(DSA_ERR_INVALID_ARG, "sel_idx: null");
    const int32_t topk = static_cast<int32_t>(sel_idx->shape[1]);
    if ((st = check_topk(topk))) return st;
    if ((st = check_sel(sel_idx, sh.T, topk))) return st;
    if ((st = check_contig(out, "out", DSA_BF16, 3, qd))) return st;
    if (!pos) return fail(DSA_ERR_INVALID_ARG, "pos: null");
    for (int t = 0; t < sh.T; ++t)
        if (pos[t] < 0 || pos[t] >= sh.L) return fail(DSA_ERR_INVALID_ARG, "pos[%d] = %d outside [0, L)", t, pos[t]);
    if (sink && !aligned16(sink)) return fail(DSA_ERR_INVALID_ARG, "sink: not 16-byte aligned");
    const Layout l = layout(sh.T, sh.L);
    if ((st = check_ws(workspace, workspace_bytes, l))) return st;
    DeviceInfo dev;
    if ((st = device_info(dev))) return st;
    StepParams p{};
    p.phases = kPhaseAttend;
    p.grid = grid_blocks(dev, false);
    set_pos(p, pos, sh.T);
    p.L = static_cast<int32_t>(sh.L);
    p.topk = topk;
    p.sel = static_cast<int32_t*>(sel_idx->data);
    p.sel_ld = sel_idx->stride[0];
    p.q = static_cast<const uint16_t*>(q->data);
    p.kv = static_cast<const uint16_t*>(kv_cache->data);
    p.kv_ld = sh.kv_ld;
    p.sink = sink;
    p.out = static_cast<uint16_t*>(out->data);
    p.err = dev.err;
    attn_params(p, workspace, l, topk);
    CUtensorMap none;
    std::memset(&none, 0, sizeof none);
    return launch(none, p, false, workspace, l, reinterpret_cast<cudaStream_t>(stream_));
}

dsa_status_t dsa_device_status(dsa_stream_t stream_)
{
    t_last_error.clear();
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream_));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    uint32_t word = 0;
    e = cudaMemcpyFromSymbol(&word, g_err_word, sizeof word);
    if (e != cudaSuccess) return cuda_fail(e, "read device error word");
    if (word) {
        const uint32_t zero = 0;
        e = cudaMemcpyToSymbol(g_err_word, &zero, sizeof zero);
        if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
        return fail(DSA_ERR_DEVICE, "device error word 0x%x (1: wait timeout, 2: bad selected index, 4: top-k state, "
                    "8: workspace control words not zero at launch, 16: device query position outside [0, L))",
                    word);
    }
    return DSA_OK;
}

const char* dsa_status_str(dsa_status_t s)
{
    switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or size";
    case DSA_ERR_CUDA: return "CUDA runtime error";
    case DSA_ERR_DEVICE: return "device-side anomaly";
    }
    return "unknown status";
}

const char* dsa_last_error(void) { return t_last_error.c_str(); }

uint64_t dsa_launch_count(void) { return g_launches.load(); }

dsa_status_t dsa_debug_fail_next_barriers(int64_t limit_cycles)
{
    t_last_error.clear();
    if (limit_cycles < 1000 || limit_cycles > kWaitLimitCycles)
        return fail(DSA_ERR_INVALID_ARG, "limit_cycles = %lld outside [1000, %lld]", (long long)limit_cycles,
                    (long long)kWaitLimitCycles);
    t_fail_barriers = limit_cycles;
    return DSA_OK;
}

void dsa_set_step_trace(void* device_buffer) { t_trace = static_cast<unsigned long long*>(device_buffer); }

int32_t dsa_step_grid(int32_t fp8_keys)
{
    DeviceInfo dev;
    if (device_info(dev)) return 0;
    return grid_blocks(dev, fp8_keys != 0);
}

void dsa_set_stage_events(void* const* events, int32_t n)
{
    if (n == 5 && events) {
        for (int i = 0; i < 5; ++i) t_stage_events[i] = events[i];
        t_stage_events_on = true;
    } else if (n == 0) {
        t_stage_events_on = false;
    }
}

}  // extern "C"
