// prolog.cu -- host side of indexer_prolog (include/dsa.h): argument checks,
// the tile / split plan, TMA descriptors and the launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>

#include "../../include/dsa.h"
#include "common.h"
#include "host.h"
#include "prolog.cuh"

using namespace dsa;
using namespace dsa::host;

namespace {

constexpr size_t kProlStatusBytes = 256;
constexpr int kGroupM = 16;

struct ProlPlan {
    int bn = 0, MT = 0, NT = 0, S = 1, Sk = 1, mk = 0, KB = 0, units = 0, grid = 0, smem = 0;
    size_t counters_off = 0, partials_off = 0, ws = 0;
};

int prolog_smem(int bn) {
    switch (bn) {
        case 32: return PrologCfg<32>::SMEM;
        case 64: return PrologCfg<64>::SMEM;
        case 128: return PrologCfg<128>::SMEM;
        default: return PrologCfg<256>::SMEM;
    }
}

// Token tile: the smallest of 32/64/128/256 that covers T (256 beyond).
// Splits: with fewer tiles than SMs, the K range is split S ways, S the largest
// count whose units still fit one wave of the SMs (one unit per CTA, so the
// weights stream at full depth and each tile's partials are added once; each
// split keeps at least 4 k-blocks, at most 16 splits).  In such a single-wave
// plan the row tile holding the key rows takes twice as many splits when they
// still fit: its epilogue is the longest, and shorter streaming hides it.
ProlPlan plan_prolog(int T, int d, int n_out, int HD, int sms) {
    ProlPlan pl;
    pl.bn = T <= 32 ? 32 : T <= 64 ? 64 : T <= 128 ? 128 : 256;
    pl.MT = (n_out + 127) / 128;
    pl.NT = (T + pl.bn - 1) / pl.bn;
    pl.KB = (d + 63) / 64;
    pl.mk = HD / 128;
    const int64_t tiles = (int64_t)pl.MT * pl.NT;
    const int smax = pl.KB / 4 < 16 ? (pl.KB / 4 < 1 ? 1 : pl.KB / 4) : 16;
    int64_t s = tiles < sms ? sms / tiles : 1;
    if (s > smax) s = smax;
    if (s < 1) s = 1;
    pl.S = (int)s;
    pl.Sk = pl.S;
    if (tiles < sms && 2 * pl.S <= smax && (tiles - pl.NT) * pl.S + (int64_t)pl.NT * 2 * pl.S <= sms) pl.Sk = 2 * pl.S;
    pl.units = (int)((tiles - pl.NT) * pl.S + (int64_t)pl.NT * pl.Sk);
    pl.grid = pl.units < sms ? pl.units : sms;
    pl.smem = prolog_smem(pl.bn);
    const int smx = pl.S > pl.Sk ? pl.S : pl.Sk;
    pl.counters_off = kProlStatusBytes;
    pl.partials_off = pl.counters_off + align256((size_t)tiles * 4);
    pl.ws = pl.partials_off + (smx > 1 ? (size_t)smx * (size_t)tiles * (size_t)pl.bn * 128 * 4 : 0);
    return pl;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

dsa_status check_prolog(const dsa_batch* bt, const dsa_prolog_inputs* pr) {
    if (!bt || bt->batch < 1 || bt->num_tokens < 1 || !bt->seq_lens || !bt->cu_q || !bt->block_table ||
        bt->max_blocks_per_seq < 1 || bt->num_blocks < 1)
        return DSA_ERR_INVALID_ARG;
    if ((int64_t)bt->num_blocks * kPage > INT32_MAX) return DSA_ERR_UNSUPPORTED;
    if (!pr || !pr->x || !pr->w_proj || !pr->k_gamma) return DSA_ERR_INVALID_ARG;
    if (pr->H_I != 8 && pr->H_I != 16 && pr->H_I != 32 && pr->H_I != 64) return DSA_ERR_UNSUPPORTED;
    if (pr->D_I != 64 && pr->D_I != 128) return DSA_ERR_UNSUPPORTED;
    if (pr->d_model < 8 || pr->d_model % 8 != 0) return DSA_ERR_UNSUPPORTED;
    if (pr->key_dtype != DSA_KEY_BF16 && pr->key_dtype != DSA_KEY_FP8_E4M3 && pr->key_dtype != DSA_KEY_MXFP8)
        return DSA_ERR_INVALID_ARG;
    if (pr->q_dtype != DSA_Q_BF16 && pr->q_dtype != DSA_Q_MXFP8) return DSA_ERR_INVALID_ARG;
    if ((pr->q_dtype == DSA_Q_MXFP8) != (pr->key_dtype == DSA_KEY_MXFP8)) return DSA_ERR_INVALID_ARG;
    if (!(pr->eps >= 0.0f)) return DSA_ERR_INVALID_ARG;
    if (pr->w_layout != DSA_W_ROW_MAJOR && pr->w_layout != DSA_W_TILE_PACKED) return DSA_ERR_INVALID_ARG;
    if (!aligned(pr->x, 16) || !aligned(pr->w_proj, 16) || !aligned(pr->k_gamma, 4)) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

template <int BN>
dsa_status launch_prolog(const dsa_batch* bt, const dsa_prolog_inputs* pr, const PrologParams& p, const ProlPlan& pl,
                         cudaStream_t stream) {
    const int n_out = p.n_out;
    CUtensorMap tm_w, tm_x;
    if (pr->w_layout == DSA_W_TILE_PACKED) {
        // [MT*KB blocks][128 rows][64 columns]: one box is one 16 KB block
        const uint64_t dims[3] = {64, 128, (uint64_t)pl.MT * pl.KB};
        const uint64_t strides[2] = {64 * 2, 128 * 64 * 2};
        const uint32_t box[3] = {64, 128, 1};
        if (!make_map(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, pr->w_proj, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return fail(DSA_ERR_CUDA, "prolog weight tensor map encoding failed");
    } else {
        const uint64_t dims[2] = {(uint64_t)pr->d_model, (uint64_t)n_out};
        const uint64_t strides[1] = {(uint64_t)pr->d_model * 2};
        const uint32_t box[2] = {64, 128};
        if (!make_map(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pr->w_proj, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return fail(DSA_ERR_CUDA, "prolog weight tensor map encoding failed");
    }
    {
        const uint64_t dims[2] = {(uint64_t)pr->d_model, (uint64_t)bt->num_tokens};
        const uint64_t strides[1] = {(uint64_t)pr->d_model * 2};
        const uint32_t box[2] = {64, (uint32_t)BN};
        if (!make_map(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pr->x, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return fail(DSA_ERR_CUDA, "prolog hidden-state tensor map encoding failed");
    }
    auto kern = &indexer_prolog_kernel<BN>;
    if (cudaError_t e = set_smem_attr(reinterpret_cast<const void*>(kern), pl.smem))
        return fail(DSA_ERR_CUDA, "prolog shared memory attribute", e);
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(pl.grid, 1, 1);
    cfg.blockDim = dim3(PrologCfg<BN>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = (size_t)pl.smem;
    cfg.stream = stream;
    if (cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p, tm_w, tm_x)) return fail(DSA_ERR_CUDA, "prolog launch", e);
    return DSA_OK;
}

}  // namespace

extern "C" {

DSA_API size_t dsa_prolog_packed_bytes(int32_t H_I, int32_t D_I, int32_t d_model) {
    if (H_I < 1 || D_I < 1 || d_model < 8 || d_model % 8 != 0) return 0;
    const int64_t n_out = (int64_t)H_I * D_I + D_I + H_I;
    return (size_t)((n_out + 127) / 128) * (size_t)((d_model + 63) / 64) * 128 * 64 * 2;
}

DSA_API dsa_status indexer_prolog_pack(const void* w_proj, void* w_packed, int32_t H_I, int32_t D_I, int32_t d_model,
                                       void* stream) {
    const size_t bytes = dsa_prolog_packed_bytes(H_I, D_I, d_model);
    if (!bytes || !w_proj || !w_packed) return fail(DSA_ERR_INVALID_ARG, "indexer_prolog_pack: invalid arguments");
    if (!aligned(w_proj, 16) || !aligned(w_packed, 16))
        return fail(DSA_ERR_INVALID_ARG, "indexer_prolog_pack: pointers must be 16-byte aligned");
    const DevInfo di = dev_info();
    if (di.sms < 1) return fail(DSA_ERR_CUDA, "indexer_prolog_pack: no device");
    const int n_out = H_I * D_I + D_I + H_I;
    const int64_t chunks = (int64_t)(bytes / 16);
    int64_t blocks = (chunks + 255) / 256;
    if (blocks > (int64_t)di.sms * 16) blocks = (int64_t)di.sms * 16;
    prolog_pack_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(w_proj), static_cast<uint4*>(w_packed), n_out, d_model, (d_model + 63) / 64, chunks);
    if (cudaError_t e = cudaGetLastError()) return fail(DSA_ERR_CUDA, "indexer_prolog_pack launch", e);
    return DSA_OK;
}

DSA_API size_t dsa_prolog_workspace_size(const dsa_batch* batch, const dsa_prolog_inputs* pr) {
    if (check_prolog(batch, pr) != DSA_OK) return 0;
    const DevInfo di = dev_info();
    if (di.sms < 1) return 0;
    const int n_out = pr->H_I * pr->D_I + pr->D_I + pr->H_I;
    return plan_prolog(batch->num_tokens, pr->d_model, n_out, pr->H_I * pr->D_I, di.sms).ws;
}

DSA_API dsa_status indexer_prolog(const dsa_batch* batch, const dsa_prolog_inputs* pr, void* q_out,
                                  uint8_t* q_scale_out, float* w_out, void* k_cache, void* k_scale, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    if (dsa_status st = check_prolog(batch, pr)) return fail(st, "indexer_prolog: invalid or unsupported arguments");
    const bool mx = pr->q_dtype == DSA_Q_MXFP8;
    if (!q_out || !w_out || !k_cache || (mx && !q_scale_out) || (pr->key_dtype != DSA_KEY_BF16 && !k_scale))
        return fail(DSA_ERR_INVALID_ARG, "indexer_prolog: missing output");
    if (!aligned(w_out, 4) || (!mx && !aligned(q_out, 2)) || (pr->key_dtype == DSA_KEY_BF16 && !aligned(k_cache, 2)) ||
        (pr->key_dtype == DSA_KEY_FP8_E4M3 && !aligned(k_scale, 4)))
        return fail(DSA_ERR_INVALID_ARG, "indexer_prolog: misaligned output");
    const DevInfo di = dev_info();
    if (di.sms < 1) return fail(DSA_ERR_CUDA, "indexer_prolog: no device");
    const int n_out = pr->H_I * pr->D_I + pr->D_I + pr->H_I;
    const ProlPlan pl = plan_prolog(batch->num_tokens, pr->d_model, n_out, pr->H_I * pr->D_I, di.sms);
    if (!workspace || workspace_bytes < pl.ws || !aligned(workspace, 256))
        return fail(DSA_ERR_WORKSPACE, "indexer_prolog: workspace missing, too small or not 256-byte aligned");
    if (pl.smem > di.max_smem) return fail(DSA_ERR_UNSUPPORTED, "indexer_prolog: shared memory");

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    PrologParams p;
    memset(&p, 0, sizeof p);
    p.gamma = pr->k_gamma;
    p.seq_lens = batch->seq_lens;
    p.cu_q = batch->cu_q;
    p.block_table = batch->block_table;
    p.q_bf16 = mx ? nullptr : static_cast<uint16_t*>(q_out);
    p.q_codes = mx ? static_cast<uint8_t*>(q_out) : nullptr;
    p.q_scale = mx ? q_scale_out : nullptr;
    p.w_out = w_out;
    p.k_bf16 = pr->key_dtype == DSA_KEY_BF16 ? static_cast<uint16_t*>(k_cache) : nullptr;
    p.k_codes = pr->key_dtype == DSA_KEY_BF16 ? nullptr : static_cast<uint8_t*>(k_cache);
    p.k_scale_f32 = pr->key_dtype == DSA_KEY_FP8_E4M3 ? static_cast<float*>(k_scale) : nullptr;
    p.k_scale_e8 = pr->key_dtype == DSA_KEY_MXFP8 ? static_cast<uint8_t*>(k_scale) : nullptr;
    p.status = reinterpret_cast<uint32_t*>(ws);
    p.counters = reinterpret_cast<uint32_t*>(ws + pl.counters_off);
    p.partials = reinterpret_cast<float*>(ws + pl.partials_off);
    p.T = batch->num_tokens;
    p.H_I = pr->H_I;
    p.D_I = pr->D_I;
    p.HD = pr->H_I * pr->D_I;
    p.n_out = n_out;
    p.B = batch->batch;
    p.max_blocks = batch->max_blocks_per_seq;
    p.num_blocks = batch->num_blocks;
    p.MT = pl.MT;
    p.NT = pl.NT;
    p.S = pl.S;
    p.Sk = pl.Sk;
    p.mk = pl.mk;
    p.KB = pl.KB;
    p.units = pl.units;
    p.group_m = kGroupM;
    p.evict_w = pl.NT == 1;
    p.w_packed = pr->w_layout == DSA_W_TILE_PACKED;
    p.eps = pr->eps;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (pl.bn) {
        case 32: return launch_prolog<32>(batch, pr, p, pl, st);
        case 64: return launch_prolog<64>(batch, pr, p, pl, st);
        case 128: return launch_prolog<128>(batch, pr, p, pl, st);
        default: return launch_prolog<256>(batch, pr, p, pl, st);
    }
}

}  // extern "C"
