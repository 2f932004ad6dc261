// idx_launch.cuh -- host launcher of the fused indexer kernel for one
// template variant: TMA descriptors for the queries and the paged key cache,
// kernel parameters, and the (cooperative, for grouped decode) launches.
// Included only by the idx_*.cu units, each of which instantiates a few
// variants, so that the variants compile in parallel.
#pragma once
#include <cstring>

#include "host.h"
#include "indexer.cuh"

namespace dsa {
namespace host {

template <bool FP8, int HI, int DI, int NQ, bool MX>
dsa_status launch_indexer(const dsa_batch* bt, const dsa_indexer_inputs* ix, int32_t* out_idx, float* out_score,
                          uint32_t* status, uint8_t* group_ws, const IdxPlan& pl, cudaStream_t stream) {
    using Cfg = IdxCfg<FP8, HI, DI, NQ, MX>;
    CUtensorMap tm_q, tm_k;
    if (MX) {
        // MXFP8 queries are read by the epilogue threads; the map (over the codes) is
        // passed but never used by a copy
        const uint64_t dims[3] = {(uint64_t)DI, (uint64_t)HI, (uint64_t)bt->num_tokens};
        const uint64_t strides[2] = {(uint64_t)DI, (uint64_t)HI * DI};
        const uint32_t box[3] = {(uint32_t)DI, (uint32_t)HI, 1};
        if (!make_map(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, ix->q_idx, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return fail(DSA_ERR_CUDA, "indexer query tensor map encoding failed");
    } else {
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
    auto kern = &indexer_topk_kernel<FP8, HI, DI, NQ, MX>;
    if (cudaError_t e = set_smem_attr(reinterpret_cast<const void*>(kern), pl.smem))
        return fail(DSA_ERR_CUDA, "indexer shared memory attribute", e);

    IndexerParams p;
    memset(&p, 0, sizeof p);
    p.seq_lens = bt->seq_lens;
    p.cu_q = bt->cu_q;
    p.block_table = bt->block_table;
    p.w = ix->w;
    p.k_scale = MX ? nullptr : ix->k_scale;
    p.k_scale_e8 = MX ? reinterpret_cast<const uint8_t*>(ix->k_scale) : nullptr;
    p.q_codes = MX ? reinterpret_cast<const uint8_t*>(ix->q_idx) : nullptr;
    p.q_scale = MX ? ix->q_scale : nullptr;
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
    p.seq_windows = pl.seq_windows;
    for (int64_t w0 = 0; w0 < pl.windows; w0 += pl.windows_per_launch) {
        p.w_begin = (int32_t)w0;
        p.w_end = (int32_t)(w0 + pl.windows_per_launch < pl.windows ? w0 + pl.windows_per_launch : pl.windows);
        if (cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p, tm_q, tm_k)) return fail(DSA_ERR_CUDA, "indexer launch", e);
    }
    return DSA_OK;
}


}  // namespace host
}  // namespace dsa
