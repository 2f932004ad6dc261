// api.cu -- host side of the C ABI declared in include/dsa.h: argument
// validation, workspace layout, TMA descriptor encoding, launch
// configuration.  Nothing here allocates device memory or synchronizes,
// except dsa_get_status.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/dsa.h"
#include "common.h"
#include "indexer.cuh"
#include "sfa.cuh"

using namespace dsa;

static_assert(sizeof(IdxMisc) <= 1024, "indexer misc block exceeds its slot");
static_assert(sizeof(SfaMisc) <= SfaCfg::MISC_BYTES, "attention misc block exceeds its slot");

namespace {

constexpr size_t kStatusBytes = 256;
constexpr int kMaxSplitTokens = 128;      // row splits are only used for fewer tokens than this
constexpr size_t kCounterBytes = kMaxSplitTokens * 2 * 2 * 4;   // split arrivals and ready counts
constexpr size_t kHeaderBytes = kStatusBytes + kCounterBytes;

// ------------------------------------------------------------------ last failure text (per host thread)
thread_local char g_last_error[256] = "";

dsa_status fail(dsa_status st, const char* what, cudaError_t e = cudaSuccess) {
    if (e != cudaSuccess)
        snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
    else
        snprintf(g_last_error, sizeof g_last_error, "%s", what);
    return st;
}

// ------------------------------------------------------------------ driver entry point (no libcuda link)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
              CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
        if (i + 1 < rank) s[i] = strides_bytes[i];
    }
    return fn(map, dt, (cuuint32_t)rank, const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DevInfo {
    int sms = 0;
    int max_smem = 0;
};

DevInfo dev_info() {
    int dev = 0;
    DevInfo di;
    if (cudaGetDevice(&dev) != cudaSuccess) return di;
    cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&di.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    return di;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dsa_status check_batch(const dsa_batch* bt) {
    if (!bt || bt->batch < 1 || bt->num_tokens < 1 || !bt->seq_lens || !bt->cu_q || !bt->block_table ||
        bt->max_blocks_per_seq < 1 || bt->num_blocks < 1 || bt->max_seq_len < 1 || bt->max_q_per_seq < 1)
        return DSA_ERR_INVALID_ARG;
    if ((int64_t)bt->max_blocks_per_seq * kPage < bt->max_seq_len) return DSA_ERR_INVALID_ARG;
    if ((int64_t)bt->num_blocks * kPage > INT32_MAX) return DSA_ERR_UNSUPPORTED;
    return DSA_OK;
}

dsa_status check_indexer(const dsa_indexer_inputs* ix) {
    if (!ix || !ix->q_idx || !ix->w || !ix->k_cache) return DSA_ERR_INVALID_ARG;
    if (ix->key_dtype != DSA_KEY_BF16 && ix->key_dtype != DSA_KEY_FP8_E4M3) return DSA_ERR_INVALID_ARG;
    if (ix->key_dtype == DSA_KEY_FP8_E4M3 && !ix->k_scale) return DSA_ERR_INVALID_ARG;
    if (ix->H_I != 8 && ix->H_I != 16 && ix->H_I != 32 && ix->H_I != 64) return DSA_ERR_UNSUPPORTED;
    if (ix->D_I != 64 && ix->D_I != 128) return DSA_ERR_UNSUPPORTED;
    if (ix->K < 1 || ix->K > kMaxTopK) return DSA_ERR_UNSUPPORTED;
    if (!aligned16(ix->q_idx) || !aligned16(ix->k_cache)) return DSA_ERR_INVALID_ARG;
    if (ix->k_scale && (reinterpret_cast<uintptr_t>(ix->k_scale) & 3u)) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

dsa_status check_attn(const dsa_attn_inputs* at) {
    if (!at || !at->q || !at->kv_cache) return DSA_ERR_INVALID_ARG;
    if (at->H < 1 || at->H > 128) return DSA_ERR_UNSUPPORTED;
    if (!aligned16(at->q) || !aligned16(at->kv_cache)) return DSA_ERR_INVALID_ARG;
    if (!(at->sm_scale > 0.0f) || at->sm_scale != at->sm_scale) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

size_t align256(size_t v);
size_t group_region_bytes(int sms);

// ------------------------------------------------------------------ indexer planning
struct IdxPlan {
    int mode = 0;        // 0 grouped decode, 1 per-token
    int nq = 1;          // kernel NQ
    int grid = 0;        // CTAs per launch
    int seqs_per_launch = 0;
    int score_cap = 0;
    int smem = 0;
    size_t group_ws = 0; // bytes of group workspace per launch
};

template <bool FP8, int HI, int DI, int NQ>
struct IdxKernel {
    using Cfg = IdxCfg<FP8, HI, DI, NQ>;
    static void* fn() { return reinterpret_cast<void*>(&indexer_topk_kernel<FP8, HI, DI, NQ>); }
};

// Fill the fields that depend on the kernel instantiation.
template <bool FP8, int HI, int DI, int NQ>
bool plan_for(const dsa_batch* bt, const DevInfo& di, IdxPlan& pl) {
    using Cfg = IdxCfg<FP8, HI, DI, NQ>;
    const int cap = (di.max_smem - Cfg::FIXED_SMEM) / 4;
    if (cap < kTileKeys * NQ) return false;
    pl.score_cap = (cap / (kTileKeys * NQ)) * (kTileKeys * NQ);
    if (pl.score_cap > kCandSlotKeys) pl.score_cap = (int)((kCandSlotKeys / (kTileKeys * NQ)) * (kTileKeys * NQ));
    pl.smem = Cfg::FIXED_SMEM + pl.score_cap * 4;
    // one CTA per SM (shared memory use allows no more); a group's select reads
    // at most 256 publication headers
    pl.grid = di.sms < 256 ? di.sms : 256;
    if (pl.mode == 1) {
        if (bt->max_seq_len > pl.score_cap) return false;
        pl.seqs_per_launch = bt->batch;
        pl.group_ws = 0;
        return true;
    }
    const int64_t mt = (bt->max_seq_len + kTileKeys - 1) / kTileKeys;   // tiles of the longest sequence
    const int64_t cap_tiles = pl.score_cap / (kTileKeys * NQ);
    // B' sequences per launch so that ceil(total/(C-B')) <= cap_tiles even if all are longest
    int64_t bp = ((int64_t)pl.grid * cap_tiles) / (mt + cap_tiles);
    if (bp > pl.grid) bp = pl.grid;
    if (bp > bt->batch) bp = bt->batch;
    while (bp >= 1 && (bp * mt + (pl.grid - bp) - 1) / (pl.grid - bp > 0 ? pl.grid - bp : 1) > cap_tiles) --bp;
    if (bp < 1) return false;
    pl.seqs_per_launch = (int)bp;
    // one stride for every NQ: the barrier words of group g sit at the same
    // offset whichever kernel used the workspace last (they are not zero
    // between calls; everything else is)
    pl.group_ws = (size_t)bp * (size_t)group_ws_bytes(2, pl.grid);
    return true;
}

using LaunchFn = dsa_status (*)(const dsa_batch*, const dsa_indexer_inputs*, int32_t*, float*, uint32_t*,
                                uint8_t*, const IdxPlan&, cudaStream_t);

template <bool FP8, int HI, int DI, int NQ>
dsa_status launch_indexer(const dsa_batch* bt, const dsa_indexer_inputs* ix, int32_t* out_idx, float* out_score,
                          uint32_t* status, uint8_t* group_ws, const IdxPlan& pl, cudaStream_t stream) {
    using Cfg = IdxCfg<FP8, HI, DI, NQ>;
    CUtensorMap tm_q, tm_k;
    {
        const uint64_t dims[3] = {(uint64_t)DI, (uint64_t)HI, (uint64_t)bt->num_tokens};
        const uint64_t strides[2] = {(uint64_t)DI * 2, (uint64_t)HI * DI * 2};
        const uint32_t box[3] = {64, (uint32_t)HI, (uint32_t)NQ};
        if (!make_map(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ix->q_idx, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return fail(DSA_ERR_CUDA, "indexer query tensor map encoding failed");
    }
    {
        const uint64_t dims[2] = {(uint64_t)DI, (uint64_t)bt->num_blocks * kPage};
        if (FP8) {
            const uint64_t strides[1] = {(uint64_t)DI};
            const uint32_t box[2] = {(uint32_t)DI, (uint32_t)kPage};
            if (!make_map(&tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, ix->k_cache, dims, strides, box,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
                return fail(DSA_ERR_CUDA, "indexer key tensor map encoding failed");
        } else {
            const uint64_t strides[1] = {(uint64_t)DI * 2};
            const uint32_t box[2] = {64, (uint32_t)kPage};
            if (!make_map(&tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ix->k_cache, dims, strides, box,
                          CU_TENSOR_MAP_SWIZZLE_128B))
                return fail(DSA_ERR_CUDA, "indexer key tensor map encoding failed");
        }
    }
    auto kern = &indexer_topk_kernel<FP8, HI, DI, NQ>;
    if (cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem))
        return fail(DSA_ERR_CUDA, "indexer shared memory attribute", e);

    IndexerParams p;
    memset(&p, 0, sizeof p);
    p.seq_lens = bt->seq_lens;
    p.cu_q = bt->cu_q;
    p.block_table = bt->block_table;
    p.w = ix->w;
    p.k_scale = ix->k_scale;
    p.out_idx = out_idx;
    p.out_score = out_score;
    p.status = status;
    p.group_ws = group_ws;
    p.group_ws_stride = group_ws_bytes(2, pl.grid);
    p.cand = reinterpret_cast<uint32_t*>(group_ws + group_region_bytes(pl.grid));
    p.cand_slot = kCandSlotKeys;
    p.B = bt->batch;
    p.T = bt->num_tokens;
    p.max_blocks = bt->max_blocks_per_seq;
    p.num_blocks = bt->num_blocks;
    p.mode = pl.mode;
    p.K = ix->K;
    p.score_cap = pl.score_cap;

    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cudaLaunchAttribute attr[1];
    cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = (size_t)pl.smem;
    cfg.stream = stream;
    if (pl.mode == 1) {
        int grid = pl.grid;
        if (grid > bt->num_tokens) grid = bt->num_tokens;
        cfg.gridDim = dim3(grid, 1, 1);
        cfg.attrs = nullptr;
        cfg.numAttrs = 0;
        p.t_begin = 0;
        p.t_end = bt->num_tokens;
        if (cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p, tm_q, tm_k)) return fail(DSA_ERR_CUDA, "indexer launch", e);
        return DSA_OK;
    }
    // grouped mode: the CTAs of a group wait for one another, so they must be
    // co-resident -- a cooperative launch guarantees it (or fails)
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(pl.grid, 1, 1);
    for (int b0 = 0; b0 < bt->batch; b0 += pl.seqs_per_launch) {
        p.b_begin = b0;
        p.b_end = b0 + pl.seqs_per_launch < bt->batch ? b0 + pl.seqs_per_launch : bt->batch;
        if (cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p, tm_q, tm_k)) return fail(DSA_ERR_CUDA, "indexer launch", e);
    }
    return DSA_OK;
}

template <bool FP8, int HI, int DI, int NQ>
bool select_impl(const dsa_batch* bt, const DevInfo& di, IdxPlan& pl, LaunchFn& fn) {
    if (!plan_for<FP8, HI, DI, NQ>(bt, di, pl)) return false;
    fn = &launch_indexer<FP8, HI, DI, NQ>;
    return true;
}

template <bool FP8, int HI, int DI>
bool select_nq(const dsa_batch* bt, const DevInfo& di, IdxPlan& pl, LaunchFn& fn) {
    if (pl.nq == 1) return select_impl<FP8, HI, DI, 1>(bt, di, pl, fn);
    return select_impl<FP8, HI, DI, 2>(bt, di, pl, fn);
}

template <bool FP8, int HI>
bool select_di(int D_I, const dsa_batch* bt, const DevInfo& di, IdxPlan& pl, LaunchFn& fn) {
    if (D_I == 64) return select_nq<FP8, HI, 64>(bt, di, pl, fn);
    return select_nq<FP8, HI, 128>(bt, di, pl, fn);
}

template <bool FP8>
bool select_hi(int H_I, int D_I, const dsa_batch* bt, const DevInfo& di, IdxPlan& pl, LaunchFn& fn) {
    switch (H_I) {
        case 8: return select_di<FP8, 8>(D_I, bt, di, pl, fn);
        case 16: return select_di<FP8, 16>(D_I, bt, di, pl, fn);
        case 32: return select_di<FP8, 32>(D_I, bt, di, pl, fn);
        default: return select_di<FP8, 64>(D_I, bt, di, pl, fn);
    }
}

dsa_status plan_indexer(const dsa_batch* bt, const dsa_indexer_inputs* ix, const DevInfo& di, IdxPlan& pl,
                        LaunchFn& fn) {
    int nq = bt->max_q_per_seq < bt->num_tokens ? bt->max_q_per_seq : bt->num_tokens;
    if (nq <= 2) {
        pl.mode = 0;
        pl.nq = nq;
    } else {
        pl.mode = 1;   // many tokens per sequence (chunked prefill): one CTA per token
        pl.nq = 1;
    }
    const bool fp8 = ix->key_dtype == DSA_KEY_FP8_E4M3;
    bool ok = fp8 ? select_hi<true>(ix->H_I, ix->D_I, bt, di, pl, fn) : select_hi<false>(ix->H_I, ix->D_I, bt, di, pl, fn);
    return ok ? DSA_OK : DSA_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ attention planning
struct AttnPlan {
    int splits = 1;
    int rows_per_split = 0;
    size_t part_bytes = 0;
};

AttnPlan plan_attn(const dsa_batch* bt, int K, const DevInfo& di) {
    AttnPlan ap;
    const int max_splits = (K + SfaCfg::ROWS - 1) / SfaCfg::ROWS;
    int s = di.sms / (2 * bt->num_tokens);
    if (s < 1 || bt->num_tokens > kMaxSplitTokens) s = 1;
    if (s > max_splits) s = max_splits;
    const int per = (K + s - 1) / s;
    ap.rows_per_split = ((per + SfaCfg::ROWS - 1) / SfaCfg::ROWS) * SfaCfg::ROWS;
    ap.splits = (K + ap.rows_per_split - 1) / ap.rows_per_split;
    if (ap.splits > 1)
        ap.part_bytes = (size_t)bt->num_tokens * ap.splits * (128 * kDv * 4 + 2 * 256 * 4);
    return ap;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Workspace layout, the same for every shape on a given device:
//   [status 256 B][split arrival counters 1 KB][indexer group region, fixed
//   size][indexer published-key slots, one per SM][attention partials]
// The indexer regions are sized for the largest grouped launch (one group per
// SM, two tokens per group), so calls of any shape sharing one workspace
// never write attention partials over the indexer's barrier words.
size_t group_region_bytes(int sms) { return align256((size_t)sms * (size_t)group_ws_bytes(2, sms)); }
size_t idx_region_bytes(const DevInfo& di) {
    return group_region_bytes(di.sms) + align256((size_t)di.sms * (size_t)kCandSlotKeys * 4);
}

dsa_status launch_attn(const dsa_batch* bt, const dsa_attn_inputs* at, const int32_t* idx, int K, void* out,
                       float* lse, uint32_t* status, uint8_t* part, const AttnPlan& ap, cudaStream_t stream) {
    CUtensorMap tm_q;
    const uint64_t dims[3] = {(uint64_t)kDqk, (uint64_t)at->H, (uint64_t)bt->num_tokens};
    const uint64_t strides[2] = {(uint64_t)kDqk * 2, (uint64_t)at->H * kDqk * 2};
    // each CTA of a pair loads its own 64 heads (heads past H read as zeros)
    const uint32_t box[3] = {64, (uint32_t)(at->H < 64 ? at->H : 64), 1};
    if (!make_map(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, at->q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return fail(DSA_ERR_CUDA, "attention query tensor map encoding failed");
    if (cudaError_t e = cudaFuncSetAttribute(&sfa_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             SfaCfg::SMEM))
        return fail(DSA_ERR_CUDA, "attention shared memory attribute", e);
    SfaParams p;
    memset(&p, 0, sizeof p);
    p.seq_lens = bt->seq_lens;
    p.cu_q = bt->cu_q;
    p.block_table = bt->block_table;
    p.kv = reinterpret_cast<const uint16_t*>(at->kv_cache);
    p.idx = idx;
    p.out = reinterpret_cast<uint16_t*>(out);
    p.lse = lse;
    p.status = status;
    p.B = bt->batch;
    p.T = bt->num_tokens;
    p.H = at->H;
    p.K = K;
    p.max_blocks = bt->max_blocks_per_seq;
    p.num_blocks = bt->num_blocks;
    p.n_splits = ap.splits;
    p.rows_per_split = ap.rows_per_split;
    p.scale_log2 = at->sm_scale * 1.4426950408889634f;
    if (ap.splits > 1) {
        p.part_o = reinterpret_cast<float*>(part);
        p.part_ml = reinterpret_cast<float*>(part + (size_t)bt->num_tokens * ap.splits * 128 * kDv * 4);
        p.split_count = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(status) + kStatusBytes);
        p.split_ready = p.split_count + kMaxSplitTokens * 2;
    }
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * bt->num_tokens * ap.splits, 1, 1);
    cfg.blockDim = dim3(SfaCfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = SfaCfg::SMEM;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaError_t e = cudaLaunchKernelEx(&cfg, &sfa_decode_kernel, p, tm_q))
        return fail(DSA_ERR_CUDA, "attention launch", e);
    return DSA_OK;
}

// ------------------------------------------------------------------ allocation-free attention
// Scratch of sparse_mla_attn_static: the status word, the split counters and
// the split partials, in module memory (zero when the module loads).  20 MiB
// holds every split plan on a 148-SM B200 (at most 74 token-splits of 258 KB).
constexpr size_t kStaticScratchBytes = size_t(20) << 20;
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of the scratch for the current device, looked up once per
// device (the first call on a device does the lookup).
uint8_t* static_scratch(dsa_status* st) {
    static std::mutex mu;
    static uint8_t* addr[64] = {};
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) {
        *st = fail(DSA_ERR_CUDA, "current device query", e);
        return nullptr;
    }
    if (dev < 0 || dev >= 64) {
        *st = fail(DSA_ERR_UNSUPPORTED, "device ordinal above 63");
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* ptr = nullptr;
        if (cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch)) {
            *st = fail(DSA_ERR_CUDA, "static scratch address lookup", e);
            return nullptr;
        }
        addr[dev] = reinterpret_cast<uint8_t*>(ptr);
    }
    return addr[dev];
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

size_t dsa_workspace_size(const dsa_batch* batch, const dsa_indexer_inputs* ix, const dsa_attn_inputs* at) {
    if (check_batch(batch) != DSA_OK) return 0;
    const DevInfo di = dev_info();
    if (di.sms <= 0) return 0;
    size_t need = kHeaderBytes + idx_region_bytes(di);
    if (ix) {
        if (check_indexer(ix) != DSA_OK) return 0;
        IdxPlan pl;
        LaunchFn fn = nullptr;
        if (plan_indexer(batch, ix, di, pl, fn) != DSA_OK) return 0;
        if (pl.group_ws > group_region_bytes(di.sms)) return 0;
    }
    if (at) {
        if (check_attn(at) != DSA_OK) return 0;
        need += align256(plan_attn(batch, kMaxTopK, di).part_bytes);
    }
    return need;
}

dsa_status indexer_topk(const dsa_batch* batch, const dsa_indexer_inputs* ix, int32_t* out_idx, float* out_score,
                        void* workspace, size_t workspace_bytes, void* stream) {
    dsa_status st = check_batch(batch);
    if (st != DSA_OK) return st;
    if ((st = check_indexer(ix)) != DSA_OK) return st;
    if (!out_idx) return DSA_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
    const DevInfo di = dev_info();
    if (di.sms <= 0) return fail(DSA_ERR_CUDA, "device query failed");
    IdxPlan pl;
    LaunchFn fn = nullptr;
    if ((st = plan_indexer(batch, ix, di, pl, fn)) != DSA_OK) return st;
    if (pl.group_ws > group_region_bytes(di.sms)) return DSA_ERR_UNSUPPORTED;
    if (workspace_bytes < kHeaderBytes + idx_region_bytes(di)) return DSA_ERR_WORKSPACE;
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    return fn(batch, ix, out_idx, out_score, reinterpret_cast<uint32_t*>(ws), ws + kHeaderBytes, pl,
              reinterpret_cast<cudaStream_t>(stream));
}

dsa_status sparse_mla_attn(const dsa_batch* batch, const dsa_attn_inputs* at, const int32_t* idx, int32_t K,
                           void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    dsa_status st = check_batch(batch);
    if (st != DSA_OK) return st;
    if ((st = check_attn(at)) != DSA_OK) return st;
    if (!idx || !out || K < 1 || K > kMaxTopK) return DSA_ERR_INVALID_ARG;
    if (!aligned16(out)) return DSA_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
    const DevInfo di = dev_info();
    if (di.sms <= 0) return fail(DSA_ERR_CUDA, "device query failed");
    if (di.max_smem < SfaCfg::SMEM) return fail(DSA_ERR_UNSUPPORTED, "device shared memory per block too small");
    const AttnPlan ap = plan_attn(batch, K, di);
    const size_t off = kHeaderBytes + idx_region_bytes(di);
    if (workspace_bytes < off + ap.part_bytes) return DSA_ERR_WORKSPACE;
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    return launch_attn(batch, at, idx, K, out, lse, reinterpret_cast<uint32_t*>(ws), ws + off, ap,
                       reinterpret_cast<cudaStream_t>(stream));
}

dsa_status sparse_mla_attn_static(const dsa_batch* batch, const dsa_attn_inputs* at, const int32_t* idx, int32_t K,
                                  void* out, float* lse, void* stream) {
    dsa_status st = check_batch(batch);
    if (st != DSA_OK) return st;
    if ((st = check_attn(at)) != DSA_OK) return st;
    if (!idx || !out || K < 1 || K > kMaxTopK) return DSA_ERR_INVALID_ARG;
    if (!aligned16(out)) return DSA_ERR_INVALID_ARG;
    const DevInfo di = dev_info();
    if (di.sms <= 0) return fail(DSA_ERR_CUDA, "device query failed");
    if (di.max_smem < SfaCfg::SMEM) return fail(DSA_ERR_UNSUPPORTED, "device shared memory per block too small");
    const AttnPlan ap = plan_attn(batch, K, di);
    const size_t need = kHeaderBytes + ap.part_bytes;
    if (need > kStaticScratchBytes) {
        snprintf(g_last_error, sizeof g_last_error,
                 "sparse_mla_attn_static: this shape needs %zu bytes of scratch, the static scratch holds %zu", need,
                 kStaticScratchBytes);
        return DSA_ERR_WORKSPACE;
    }
    uint8_t* ws = static_scratch(&st);
    if (!ws) return st;
    return launch_attn(batch, at, idx, K, out, lse, reinterpret_cast<uint32_t*>(ws), ws + kHeaderBytes, ap,
                       reinterpret_cast<cudaStream_t>(stream));
}

dsa_status dsa_decode(const dsa_batch* batch, const dsa_indexer_inputs* ix, const dsa_attn_inputs* at,
                      int32_t* out_idx, float* out_score, void* out, float* lse, void* workspace,
                      size_t workspace_bytes, void* stream) {
    dsa_status st = check_batch(batch);
    if (st != DSA_OK) return st;
    if ((st = check_indexer(ix)) != DSA_OK) return st;
    if ((st = check_attn(at)) != DSA_OK) return st;
    if (!out_idx || !out) return DSA_ERR_INVALID_ARG;
    const size_t need = dsa_workspace_size(batch, ix, at);
    if (need == 0) return DSA_ERR_UNSUPPORTED;
    if (workspace_bytes < need) return DSA_ERR_WORKSPACE;
    st = indexer_topk(batch, ix, out_idx, out_score, workspace, workspace_bytes, stream);
    if (st != DSA_OK) return st;
    return sparse_mla_attn(batch, at, out_idx, ix->K, out, lse, workspace, workspace_bytes, stream);
}

dsa_status dsa_get_status(void* workspace, void* stream, int32_t* device_status) {
    if (!workspace || !device_status) return DSA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    if (cudaError_t e = cudaStreamSynchronize(s)) return fail(DSA_ERR_CUDA, "stream synchronize", e);
    if (cudaError_t e = cudaMemcpy(&v, workspace, sizeof v, cudaMemcpyDeviceToHost))
        return fail(DSA_ERR_CUDA, "status read", e);
    const uint32_t zero = 0;
    if (v != 0)
        if (cudaError_t e = cudaMemcpy(workspace, &zero, sizeof zero, cudaMemcpyHostToDevice))
            return fail(DSA_ERR_CUDA, "status clear", e);
    *device_status = (int32_t)v;
    return DSA_OK;
}

int32_t dsa_decode_launch_count(const dsa_batch* batch, const dsa_indexer_inputs* ix, const dsa_attn_inputs* at) {
    if (check_batch(batch) != DSA_OK || check_indexer(ix) != DSA_OK || check_attn(at) != DSA_OK) return -1;
    const DevInfo di = dev_info();
    if (di.sms <= 0) return -1;
    IdxPlan pl;
    LaunchFn fn = nullptr;
    if (plan_indexer(batch, ix, di, pl, fn) != DSA_OK) return -1;
    const int idx_launches = pl.mode == 1 ? 1 : (batch->batch + pl.seqs_per_launch - 1) / pl.seqs_per_launch;
    const AttnPlan ap = plan_attn(batch, ix->K, di);
    (void)ap;   // the split merge runs inside the attention kernel
    return idx_launches + 1;
}

const char* dsa_status_str(int32_t s) {
    switch (s) {
        case DSA_OK: return "ok";
        case DSA_ERR_INVALID_ARG: return "invalid argument";
        case DSA_ERR_UNSUPPORTED: return "unsupported shape or configuration";
        case DSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case DSA_ERR_CUDA: return "CUDA call failed";
        case DSA_ERR_TIMEOUT: return "device wait timed out";
        case DSA_ERR_DEVICE_BOUNDS: return "device saw an out-of-range block id or index";
        case DSA_ERR_CAPACITY: return "key chunk exceeded on-chip capacity";
        default: return "unknown status";
    }
}

const char* dsa_last_error(void) { return g_last_error; }

const char* dsa_version(void) { return "dsa-b200 0.1.0 (sm_100a)"; }

#ifdef DSA_TRACE
// Tracing builds only: copy the per-CTA %globaltimer table ([2048][16] u64).
DSA_API int32_t dsa_trace_read(void* host_dst, size_t bytes) {
    if (bytes > sizeof(g_dsa_trace)) bytes = sizeof(g_dsa_trace);
    return cudaMemcpyFromSymbol(host_dst, g_dsa_trace, bytes) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}
DSA_API int32_t dsa_trace_blk_read(void* host_dst, size_t bytes) {
    if (bytes > sizeof(g_dsa_trace_blk)) bytes = sizeof(g_dsa_trace_blk);
    return cudaMemcpyFromSymbol(host_dst, g_dsa_trace_blk, bytes) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}
#endif

}  // extern "C"
