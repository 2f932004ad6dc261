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
#include "host.h"
#include "indexer.cuh"
#include "kvfp8.cuh"
#include "sfa.cuh"

using namespace dsa;
using namespace dsa::host;

static_assert(sizeof(IdxMisc) <= 1024, "indexer misc block exceeds its slot");
static_assert(sizeof(SfaMisc) <= SfaCfg::MISC_BYTES, "attention misc block exceeds its slot");

namespace {

// Status area at the start of every workspace: word 0 = device status, word 1 =
// bounded-wait limit in microseconds (0: the 1 s default), word 2 = fault
// injection bits (test hooks; zero in normal use).
constexpr size_t kStatusBytes = 256;
constexpr size_t kHeaderBytes = kStatusBytes;


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
    if (ix->key_dtype != DSA_KEY_BF16 && ix->key_dtype != DSA_KEY_FP8_E4M3 && ix->key_dtype != DSA_KEY_MXFP8)
        return DSA_ERR_INVALID_ARG;
    if (ix->key_dtype != DSA_KEY_BF16 && !ix->k_scale) return DSA_ERR_INVALID_ARG;
    if (ix->q_dtype != DSA_Q_BF16 && ix->q_dtype != DSA_Q_MXFP8) return DSA_ERR_INVALID_ARG;
    // MXFP8 queries and MXFP8 keys go together (the indexer's Q and K are both quantized)
    if ((ix->q_dtype == DSA_Q_MXFP8) != (ix->key_dtype == DSA_KEY_MXFP8)) return DSA_ERR_INVALID_ARG;
    if (ix->q_dtype == DSA_Q_MXFP8 && !ix->q_scale) return DSA_ERR_INVALID_ARG;
    // MXFP8 key scales arrive by 16-byte aligned bulk copies, one per page
    if (ix->key_dtype == DSA_KEY_MXFP8 && !aligned16(ix->k_scale)) return DSA_ERR_INVALID_ARG;
    if (ix->H_I != 8 && ix->H_I != 16 && ix->H_I != 32 && ix->H_I != 64) return DSA_ERR_UNSUPPORTED;
    if (ix->D_I != 64 && ix->D_I != 128) return DSA_ERR_UNSUPPORTED;
    if (ix->K < 1 || ix->K > kMaxTopK) return DSA_ERR_UNSUPPORTED;
    if (!aligned16(ix->q_idx) || !aligned16(ix->k_cache)) return DSA_ERR_INVALID_ARG;
    if (ix->key_dtype == DSA_KEY_FP8_E4M3 && (reinterpret_cast<uintptr_t>(ix->k_scale) & 3u)) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

dsa_status check_attn(const dsa_attn_inputs* at) {
    if (!at || !at->q || !at->kv_cache) return DSA_ERR_INVALID_ARG;
    if (at->H < 1 || at->H > 128) return DSA_ERR_UNSUPPORTED;
    if (!aligned16(at->q) || !aligned16(at->kv_cache)) return DSA_ERR_INVALID_ARG;
    if (at->kv_dtype != DSA_KV_BF16 && at->kv_dtype != DSA_KV_FP8) return DSA_ERR_INVALID_ARG;
    if (at->kv_dtype == DSA_KV_FP8 && (!at->kv_scale || (reinterpret_cast<uintptr_t>(at->kv_scale) & 3u)))
        return DSA_ERR_INVALID_ARG;
    if (!(at->sm_scale > 0.0f) || at->sm_scale != at->sm_scale) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}


// ------------------------------------------------------------------ indexer planning
// Fill the fields that depend on the kernel instantiation.
template <bool FP8, int HI, int DI, int NQ, bool MX>
bool plan_for(const dsa_batch* bt, const DevInfo& di, IdxPlan& pl) {
    using Cfg = IdxCfg<FP8, HI, DI, NQ, MX>;
    const int cap = (di.max_smem - Cfg::FIXED_SMEM) / 4;
    if (cap < kTileKeys * NQ) return false;
    pl.score_cap = (cap / (kTileKeys * NQ)) * (kTileKeys * NQ);
    if (pl.score_cap > kCandSlotKeys) pl.score_cap = (int)((kCandSlotKeys / (kTileKeys * NQ)) * (kTileKeys * NQ));
    pl.smem = Cfg::FIXED_SMEM + pl.score_cap * 4;
    // one CTA per SM (shared memory use allows no more); a group's select reads
    // at most 256 publication headers
    pl.grid = di.sms < 256 ? di.sms : 256;
    // a work item's page ids are staged in shared memory (MAX_PAGES of them)
    constexpr int64_t kMaxItemKeys = (int64_t)Cfg::MAX_PAGES * kPage;
    if (pl.mode == 1) {
        if (bt->max_seq_len > pl.score_cap || bt->max_seq_len > kMaxItemKeys) return false;
        pl.group_ws = 0;
        return true;
    }
    const int64_t mt = (bt->max_seq_len + kTileKeys - 1) / kTileKeys;   // tiles of the longest window
    int64_t cap_tiles = pl.score_cap / (kTileKeys * NQ);
    if (cap_tiles > kMaxItemKeys / kTileKeys) cap_tiles = kMaxItemKeys / kTileKeys;
    // W' windows per launch so that ceil(total/(C-W')) <= cap_tiles even if all are longest
    int64_t bp = ((int64_t)pl.grid * cap_tiles) / (mt + cap_tiles);
    if (bp > pl.grid) bp = pl.grid;
    if (bp > pl.windows) bp = pl.windows;
    while (bp >= 1 && (bp * mt + (pl.grid - bp) - 1) / (pl.grid - bp > 0 ? pl.grid - bp : 1) > cap_tiles) --bp;
    if (bp < 1) return false;
    pl.windows_per_launch = (int)bp;
    // one stride for every NQ: the barrier words of group g sit at the same
    // offset whichever kernel used the workspace last (they are not zero
    // between calls; everything else is)
    pl.group_ws = (size_t)bp * (size_t)group_ws_bytes(2, pl.grid);
    return true;
}

template <bool FP8, int HI, int DI, int NQ, bool MX>
bool select_impl(const dsa_batch* bt, const DevInfo& di, IdxPlan& pl, LaunchFn& fn) {
    if (!plan_for<FP8, HI, DI, NQ, MX>(bt, di, pl)) return false;
    fn = &launch_indexer<FP8, HI, DI, NQ, MX>;
    return true;
}

template <bool FP8, int HI, int DI, bool MX>
bool select_nq(const dsa_batch* bt, const DevInfo& di, IdxPlan& pl, LaunchFn& fn) {
    if (pl.nq == 1) return select_impl<FP8, HI, DI, 1, MX>(bt, di, pl, fn);
    return select_impl<FP8, HI, DI, 2, MX>(bt, di, pl, fn);
}

template <bool FP8, int HI, bool MX>
bool select_di(int D_I, const dsa_batch* bt, const DevInfo& di, IdxPlan& pl, LaunchFn& fn) {
    if (D_I == 64) return select_nq<FP8, HI, 64, MX>(bt, di, pl, fn);
    return select_nq<FP8, HI, 128, MX>(bt, di, pl, fn);
}

template <bool FP8, bool MX>
bool select_hi(int H_I, int D_I, const dsa_batch* bt, const DevInfo& di, IdxPlan& pl, LaunchFn& fn) {
    switch (H_I) {
        case 8: return select_di<FP8, 8, MX>(D_I, bt, di, pl, fn);
        case 16: return select_di<FP8, 16, MX>(D_I, bt, di, pl, fn);
        case 32: return select_di<FP8, 32, MX>(D_I, bt, di, pl, fn);
        default: return select_di<FP8, 64, MX>(D_I, bt, di, pl, fn);
    }
}

// Up to two query tokens per sequence (decode, speculative verify): grouped mode,
// one window per sequence.  More (chunked prefill, longer verify): one CTA per
// token when a token's whole score row fits one CTA's shared memory; otherwise
// grouped mode over windows of two tokens, each window split over enough CTAs.
dsa_status plan_indexer(const dsa_batch* bt, const dsa_indexer_inputs* ix, const DevInfo& di, IdxPlan& pl,
                        LaunchFn& fn) {
    const int nq = bt->max_q_per_seq < bt->num_tokens ? bt->max_q_per_seq : bt->num_tokens;
    auto select = [&]() {
        switch (ix->key_dtype) {
            case DSA_KEY_FP8_E4M3: return select_hi<true, false>(ix->H_I, ix->D_I, bt, di, pl, fn);
            case DSA_KEY_MXFP8: return select_hi<true, true>(ix->H_I, ix->D_I, bt, di, pl, fn);
            default: return select_hi<false, false>(ix->H_I, ix->D_I, bt, di, pl, fn);
        }
    };
    if (nq <= 2) {
        pl.mode = 0;
        pl.nq = nq;
        pl.seq_windows = 1;
        pl.windows = bt->batch;
        return select() ? DSA_OK : DSA_ERR_UNSUPPORTED;
    }
    pl.mode = 1;
    pl.nq = 1;
    if (select()) return DSA_OK;
    // sum_b ceil(nq_b / 2) <= min(B * ceil(max_q / 2), T / 2 + B): launches past the
    // last window find no work
    pl.mode = 0;
    pl.nq = 2;
    pl.seq_windows = 0;
    const int64_t by_max = (int64_t)bt->batch * ((nq + 1) / 2);
    const int64_t by_total = (int64_t)(bt->num_tokens + 1) / 2 + bt->batch;
    pl.windows = by_max < by_total ? by_max : by_total;
    return select() ? DSA_OK : DSA_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ attention planning
// The selected rows of all tokens form T * ceil(K/64) blocks of 64 rows; each
// two-CTA cluster ("pair") of the grid takes a contiguous range of them.
struct AttnPlan {
    int pairs = 1;
    int align_tokens = 0;       // pairs take whole tokens (no token is shared, nothing to merge)
    int64_t total_blocks = 0;
    bool combine = false;       // some token is shared by several pairs: the merge kernel runs
    size_t slot_bytes = 0;      // partial slots, [SM pairs][2 sides][2 CTAs], the same for every shape
};

// With many more tokens than SM pairs (at least kAlignTokens per pair), every
// pair takes whole tokens: the ranges differ by at most one token, and nothing
// is merged.  Otherwise the blocks are shared evenly by min(SM pairs, blocks)
// pairs, so every pair streams the same number of rows, and the tokens cut by
// a range boundary are merged by the second kernel.
AttnPlan plan_attn(const dsa_batch* bt, int K, const DevInfo& di) {
    constexpr int64_t kAlignTokens = 8;
    AttnPlan ap;
    const int nb = (K + SfaCfg::ROWS - 1) / SfaCfg::ROWS;
    const int64_t T = bt->num_tokens;
    ap.total_blocks = T * nb;
    const int pmax = di.sms / 2 > 0 ? di.sms / 2 : 1;
    if (T >= kAlignTokens * pmax) {
        ap.pairs = pmax;
        ap.align_tokens = 1;
    } else {
        ap.pairs = (int)(ap.total_blocks < pmax ? ap.total_blocks : pmax);
        // a token is shared when a range boundary falls inside it
        for (int pr = 1; pr < ap.pairs && !ap.combine; ++pr)
            ap.combine = (ap.total_blocks * pr / ap.pairs) % nb != 0;
    }
    ap.slot_bytes = (size_t)pmax * 2 * 2 * (size_t)SfaCfg::SLOT_BYTES;
    return ap;
}

// Workspace layout, the same for every shape on a given device:
//   [status 256 B][indexer group region, fixed size][indexer published-key
//   slots, one per SM][attention partial slots]
// The indexer regions are sized for the largest grouped launch (one group per
// SM, two tokens per group), so calls of any shape sharing one workspace
// never write attention partials over the indexer's barrier words.
size_t idx_region_bytes(const DevInfo& di) {
    return group_region_bytes(di.sms) + align256((size_t)di.sms * (size_t)kCandSlotKeys * 4);
}

dsa_status launch_attn(const dsa_batch* bt, const dsa_attn_inputs* at, const int32_t* idx, int K, void* out,
                       float* lse, uint32_t* status, uint8_t* attn_ws, const AttnPlan& ap, cudaStream_t stream,
                       bool dependent, bool early_q) {
    CUtensorMap tm_q;
    const uint64_t dims[3] = {(uint64_t)kDqk, (uint64_t)at->H, (uint64_t)bt->num_tokens};
    const uint64_t strides[2] = {(uint64_t)kDqk * 2, (uint64_t)at->H * kDqk * 2};
    // each CTA of a pair loads its own 64 heads (heads past H read as zeros)
    const uint32_t box[3] = {64, (uint32_t)(at->H < 64 ? at->H : 64), 1};
    if (!make_map(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, at->q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return fail(DSA_ERR_CUDA, "attention query tensor map encoding failed");
    // latent cache as [rows, 576] with one-row boxes of 64 columns, 128-byte swizzle: the
    // kernel's row gathers (tile::gather4) fetch four rows of one box each
    CUtensorMap tm_kv;
    {
        const uint64_t kdims[2] = {(uint64_t)kDqk, (uint64_t)bt->num_blocks * kPage};
        const uint64_t kstrides[1] = {(uint64_t)kDqk * 2};
        const uint32_t kbox[2] = {64, 1};
        if (!make_map(&tm_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, at->kv_cache, kdims, kstrides, kbox,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return fail(DSA_ERR_CUDA, "latent cache tensor map encoding failed");
    }
    if (cudaError_t e = set_smem_attr(reinterpret_cast<const void*>(&sfa_decode_kernel), SfaCfg::SMEM))
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
    p.scale_log2 = at->sm_scale * 1.4426950408889634f;
    p.early_q = early_q ? 1 : 0;
    p.align_tokens = ap.align_tokens;
    p.part = attn_ws;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // a programmatic dependent of the preceding launch (the indexer, in
    // dsa_decode): the kernel waits for it with griddepcontrol.wait before
    // reading the index list, and runs its prologue while it finishes
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(2 * ap.pairs, 1, 1);
    cfg.blockDim = dim3(SfaCfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = SfaCfg::SMEM;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 2 : 1;
    if (cudaError_t e = cudaLaunchKernelEx(&cfg, &sfa_decode_kernel, p, tm_q, tm_kv))
        return fail(DSA_ERR_CUDA, "attention launch", e);
    if (!ap.combine) return DSA_OK;
    // the merge of shared tokens: a programmatic dependent of the attention launch
    // (scheduled early, it waits for that grid before reading the partials)
    cudaLaunchConfig_t ccfg;
    memset(&ccfg, 0, sizeof ccfg);
    ccfg.gridDim = dim3((unsigned)bt->num_tokens, (unsigned)((at->H + 7) / 8), 1);
    ccfg.blockDim = dim3(SfaCfg::COMBINE_THREADS, 1, 1);
    ccfg.stream = stream;
    ccfg.attrs = &attr[1];
    ccfg.numAttrs = 1;
    if (cudaError_t e = cudaLaunchKernelEx(&ccfg, &sfa_combine_kernel, p, ap.pairs))
        return fail(DSA_ERR_CUDA, "attention merge launch", e);
    return DSA_OK;
}

// ------------------------------------------------------------------ FP8 latent cache
// The selected rows of up to kFp8ChunkTokens tokens at a time are dequantized
// into a bf16 staging area of the workspace, then the attention runs over them
// through a staging batch (one sequence per token; see kvfp8.cuh).
constexpr int kFp8ChunkTokens = 64;

struct Fp8Stage {
    int tc = 0, KP = 0;
    size_t stage_bytes = 0, lens_off = 0, cu_off = 0, table_off = 0, idx_off = 0, total = 0;
};

Fp8Stage fp8_stage_layout(int64_t T, int K) {
    Fp8Stage f;
    f.tc = (int)(T < kFp8ChunkTokens ? T : kFp8ChunkTokens);
    f.KP = (K + kPage - 1) / kPage * kPage;
    f.stage_bytes = align256((size_t)f.tc * f.KP * kDqk * 2);
    f.lens_off = f.stage_bytes;
    f.cu_off = f.lens_off + align256((size_t)f.tc * 4);
    f.table_off = f.cu_off + align256((size_t)(f.tc + 1) * 4);
    f.idx_off = f.table_off + align256((size_t)f.tc * (f.KP / kPage) * 4);
    f.total = f.idx_off + align256((size_t)f.tc * K * 4);
    return f;
}

// Attention over an FP8 latent cache, chunk by chunk.  The first staging launch is
// a plain stream-ordered launch (after the indexer, in dsa_decode); each attention
// launch is a programmatic dependent of its staging launch.
dsa_status launch_attn_fp8(const dsa_batch* bt, const dsa_attn_inputs* at, const int32_t* idx, int K, void* out,
                           float* lse, uint32_t* status, uint8_t* attn_ws, uint8_t* stage_ws, const DevInfo& di,
                           cudaStream_t stream) {
    const int64_t T = bt->num_tokens;
    const Fp8Stage f = fp8_stage_layout(T, K);
    for (int64_t t0 = 0; t0 < T; t0 += f.tc) {
        const int tc = (int)(T - t0 < f.tc ? T - t0 : f.tc);
        KvStageParams kp;
        memset(&kp, 0, sizeof kp);
        kp.seq_lens = bt->seq_lens;
        kp.cu_q = bt->cu_q;
        kp.block_table = bt->block_table;
        kp.kv_codes = static_cast<const uint8_t*>(at->kv_cache);
        kp.kv_scale = at->kv_scale;
        kp.idx = idx;
        kp.stage = reinterpret_cast<uint16_t*>(stage_ws);
        kp.s_seq_lens = reinterpret_cast<int32_t*>(stage_ws + f.lens_off);
        kp.s_cu_q = reinterpret_cast<int32_t*>(stage_ws + f.cu_off);
        kp.s_table = reinterpret_cast<int32_t*>(stage_ws + f.table_off);
        kp.s_idx = reinterpret_cast<int32_t*>(stage_ws + f.idx_off);
        kp.status = status;
        kp.B = bt->batch;
        kp.max_blocks = bt->max_blocks_per_seq;
        kp.num_blocks = bt->num_blocks;
        kp.K = K;
        kp.KP = f.KP;
        kp.t0 = (int32_t)t0;
        kp.tc = tc;
        const int rows_per_block = kKvRowsPerWarp * kKvStageWarps;
        const dim3 grid((unsigned)((K + rows_per_block - 1) / rows_per_block), (unsigned)tc, 1);
        kv_fp8_stage_kernel<<<grid, 32 * kKvStageWarps, 0, stream>>>(kp);
        if (cudaError_t e = cudaGetLastError()) return fail(DSA_ERR_CUDA, "latent staging launch", e);
        // the chunk's tokens as sequences of their own staged rows
        dsa_batch sb;
        memset(&sb, 0, sizeof sb);
        sb.batch = tc;
        sb.num_tokens = tc;
        sb.seq_lens = kp.s_seq_lens;
        sb.cu_q = kp.s_cu_q;
        sb.block_table = kp.s_table;
        sb.max_blocks_per_seq = f.KP / kPage;
        sb.num_blocks = tc * (f.KP / kPage);
        sb.max_seq_len = f.KP;
        sb.max_q_per_seq = 1;
        dsa_attn_inputs sa = *at;
        sa.q = static_cast<const uint8_t*>(at->q) + t0 * at->H * kDqk * 2;
        sa.kv_cache = stage_ws;
        sa.kv_dtype = DSA_KV_BF16;
        sa.kv_scale = nullptr;
        const AttnPlan ap = plan_attn(&sb, K, di);
        void* o = static_cast<uint8_t*>(out) + t0 * at->H * kDv * 2;
        float* l = lse ? lse + t0 * at->H : nullptr;
        if (dsa_status st = launch_attn(&sb, &sa, kp.s_idx, K, o, l, status, attn_ws, ap, stream, true, true))
            return st;
    }
    return DSA_OK;
}

int64_t fp8_launches(const dsa_batch* bt, int K, const DevInfo& di) {
    const Fp8Stage f = fp8_stage_layout(bt->num_tokens, K);
    int64_t n = 0;
    for (int64_t t0 = 0; t0 < bt->num_tokens; t0 += f.tc) {
        const int tc = (int)(bt->num_tokens - t0 < f.tc ? bt->num_tokens - t0 : f.tc);
        dsa_batch sb = *bt;
        sb.batch = tc;
        sb.num_tokens = tc;
        n += 2 + (plan_attn(&sb, K, di).combine ? 1 : 0);
    }
    return n;
}

// ------------------------------------------------------------------ allocation-free attention
// Scratch of sparse_mla_attn_static, in module memory: the status area and the
// partial slots of tokens shared by several CTA pairs.  20 MiB holds the
// largest plan of a 148-SM B200 (74 pairs x 2 sides x 2 CTAs x 66 KB of slots
// = 19.5 MB), for any token count.  Every GPU that loads the library holds it
// until exit.
constexpr size_t kStaticScratchBytes = size_t(20) << 20;
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// Device address of the scratch for the current device and context.  The
// lookup (cudaGetSymbolAddress, with the device current) is made by the first
// call on a device and made again only if that device's context changed
// (e.g. after cudaDeviceReset the module is loaded at a new address).
uint8_t* static_scratch(dsa_status* st) {
    static std::mutex mu;
    static uint8_t* addr[kMaxDevices] = {};
    static CUcontext ctx_of[kMaxDevices] = {};
    static CtxGetCurrentFn ctx_fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* fp = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fp, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            ctx_fn = reinterpret_cast<CtxGetCurrentFn>(fp);
    });
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) {
        *st = fail(DSA_ERR_CUDA, "current device query", e);
        return nullptr;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        *st = fail(DSA_ERR_UNSUPPORTED, "device ordinal above 63");
        return nullptr;
    }
    // the runtime makes the device's primary context current on first use
    if (cudaError_t e = cudaFree(nullptr)) {
        *st = fail(DSA_ERR_CUDA, "context initialisation", e);
        return nullptr;
    }
    CUcontext ctx = nullptr;
    if (ctx_fn) ctx_fn(&ctx);
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev] || ctx_of[dev] != ctx) {
        void* ptr = nullptr;
        if (cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch)) {
            *st = fail(DSA_ERR_CUDA, "static scratch address lookup", e);
            return nullptr;
        }
        addr[dev] = reinterpret_cast<uint8_t*>(ptr);
        ctx_of[dev] = ctx;
    }
    return addr[dev];
}

// Attention part of a workspace: the partial slots.
size_t attn_region_bytes(const AttnPlan& ap) { return align256(ap.slot_bytes); }

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
        // sized for the largest Top-K, so one workspace serves any K
        need += attn_region_bytes(plan_attn(batch, kMaxTopK, di));
        if (at->kv_dtype == DSA_KV_FP8) need += fp8_stage_layout(batch->num_tokens, ix ? ix->K : kMaxTopK).total;
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
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    if (at->kv_dtype == DSA_KV_FP8) {
        const size_t aoff = off + attn_region_bytes(plan_attn(batch, kMaxTopK, di));
        if (workspace_bytes < aoff + fp8_stage_layout(batch->num_tokens, K).total) return DSA_ERR_WORKSPACE;
        return launch_attn_fp8(batch, at, idx, K, out, lse, reinterpret_cast<uint32_t*>(ws), ws + off, ws + aoff, di,
                               reinterpret_cast<cudaStream_t>(stream));
    }
    if (workspace_bytes < off + attn_region_bytes(ap)) return DSA_ERR_WORKSPACE;
    return launch_attn(batch, at, idx, K, out, lse, reinterpret_cast<uint32_t*>(ws), ws + off, ap,
                       reinterpret_cast<cudaStream_t>(stream), true, false);
}

dsa_status sparse_mla_attn_static(const dsa_batch* batch, const dsa_attn_inputs* at, const int32_t* idx, int32_t K,
                                  void* out, float* lse, void* stream) {
    dsa_status st = check_batch(batch);
    if (st != DSA_OK) return st;
    if ((st = check_attn(at)) != DSA_OK) return st;
    if (!idx || !out || K < 1 || K > kMaxTopK) return DSA_ERR_INVALID_ARG;
    if (!aligned16(out)) return DSA_ERR_INVALID_ARG;
    if (at->kv_dtype != DSA_KV_BF16)
        return fail(DSA_ERR_UNSUPPORTED, "sparse_mla_attn_static: the FP8 latent cache needs a caller workspace");
    const DevInfo di = dev_info();
    if (di.sms <= 0) return fail(DSA_ERR_CUDA, "device query failed");
    if (di.max_smem < SfaCfg::SMEM) return fail(DSA_ERR_UNSUPPORTED, "device shared memory per block too small");
    const AttnPlan ap = plan_attn(batch, K, di);
    const size_t need = kHeaderBytes + attn_region_bytes(ap);
    if (need > kStaticScratchBytes) {
        char msg[160];
        snprintf(msg, sizeof msg,
                 "sparse_mla_attn_static: this shape needs %zu bytes of scratch, the static scratch holds %zu", need,
                 kStaticScratchBytes);
        set_last_error(msg);
        return DSA_ERR_WORKSPACE;
    }
    uint8_t* ws = static_scratch(&st);
    if (!ws) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // every call starts from a clean status area (the test-hook words included), so a
    // call that ended in a device error cannot leave stale state to later calls
    if (cudaError_t e = cudaMemsetAsync(ws, 0, kHeaderBytes, s))
        return fail(DSA_ERR_CUDA, "static scratch clear", e);
    return launch_attn(batch, at, idx, K, out, lse, reinterpret_cast<uint32_t*>(ws), ws + kHeaderBytes, ap, s,
                       false, false);
}

dsa_status dsa_decode(const dsa_batch* batch, const dsa_indexer_inputs* ix, const dsa_attn_inputs* at,
                      int32_t* out_idx, float* out_score, void* out, float* lse, void* workspace,
                      size_t workspace_bytes, void* stream) {
    dsa_status st = check_batch(batch);
    if (st != DSA_OK) return st;
    if ((st = check_indexer(ix)) != DSA_OK) return st;
    if ((st = check_attn(at)) != DSA_OK) return st;
    if (!out_idx || !out) return DSA_ERR_INVALID_ARG;
    if (!aligned16(out)) return DSA_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
    const DevInfo di = dev_info();
    if (di.sms <= 0) return fail(DSA_ERR_CUDA, "device query failed");
    if (di.max_smem < SfaCfg::SMEM) return fail(DSA_ERR_UNSUPPORTED, "device shared memory per block too small");
    // one plan for each stage, one workspace layout
    IdxPlan pl;
    LaunchFn fn = nullptr;
    if ((st = plan_indexer(batch, ix, di, pl, fn)) != DSA_OK) return st;
    if (pl.group_ws > group_region_bytes(di.sms)) return DSA_ERR_UNSUPPORTED;
    const AttnPlan ap = plan_attn(batch, ix->K, di);
    const size_t off = kHeaderBytes + idx_region_bytes(di);
    const size_t aoff = off + attn_region_bytes(plan_attn(batch, kMaxTopK, di));
    if (workspace_bytes < off + attn_region_bytes(ap)) return DSA_ERR_WORKSPACE;
    if (at->kv_dtype == DSA_KV_FP8 && workspace_bytes < aoff + fp8_stage_layout(batch->num_tokens, ix->K).total)
        return DSA_ERR_WORKSPACE;
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = fn(batch, ix, out_idx, out_score, reinterpret_cast<uint32_t*>(ws), ws + kHeaderBytes, pl, s);
    if (st != DSA_OK) return st;
    if (at->kv_dtype == DSA_KV_FP8)
        return launch_attn_fp8(batch, at, out_idx, ix->K, out, lse, reinterpret_cast<uint32_t*>(ws), ws + off, ws + aoff,
                               di, s);
    // the attention launch depends programmatically on the indexer launch just made
    return launch_attn(batch, at, out_idx, ix->K, out, lse, reinterpret_cast<uint32_t*>(ws), ws + off, ap, s, true,
                       true);
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
    const int64_t n_idx = pl.mode == 1 ? 1 : idx_launches(pl.windows, pl.windows_per_launch);
    if (at->kv_dtype == DSA_KV_FP8) return (int32_t)(n_idx + fp8_launches(batch, ix->K, di));   // staging + attention per chunk
    return (int32_t)n_idx + 1 + (plan_attn(batch, ix->K, di).combine ? 1 : 0);   // attention (+ merge)
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

const char* dsa_last_error(void) { return last_error_text(); }

const char* dsa_version(void) { return "dsa-b200 0.1.0 (sm_100a)"; }



}  // extern "C"
