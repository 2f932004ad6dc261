// kvfp8.cuh -- the FP8 latent cache for sparse attention: a gather kernel that
// reads the selected rows of an e4m3 latent cache (one fp32 scale per 128
// elements of a row, "Day0 Adaptation and Performance Optimization for Novel
// Long-Sequence Reasoning Models", section 4: FP8 KV cache quantized per token
// and per head in tiles of 128; "Large Model Inference Acceleration ...",
// section 2.2), multiplies each code by its tile's scale and stores the rows as
// bf16 in a staging area, token-major, K rows per token.  The sparse attention
// kernel then runs unchanged over the staged rows, through a batch in which each
// token is a sequence of its own staged rows (written here too): token i's
// block-table row lists its own pages of the staging area, its selected
// positions become 0..K-1 (-1 where the index list has -1).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "common.h"

namespace dsa {

struct KvStageParams {
    const int32_t* seq_lens;    // the step's batch
    const int32_t* cu_q;
    const int32_t* block_table;
    const uint8_t* kv_codes;    // [num_blocks*64, 576] e4m3 codes
    const float* kv_scale;      // [num_blocks*64, 5] fp32 tile scales
    const int32_t* idx;         // [T, K] selected positions
    uint16_t* stage;            // [tc * KP, 576] bf16 rows of the chunk's tokens
    int32_t* s_seq_lens;        // the staging batch: [tc]
    int32_t* s_cu_q;            // [tc + 1]
    int32_t* s_table;           // [tc, KP / 64]
    int32_t* s_idx;             // [tc, K]
    uint32_t* status;
    int32_t B, max_blocks, num_blocks, K, KP, t0, tc;
};

constexpr int kKvTiles = 5;                 // 4 latent tiles of 128 + the 64-element RoPE tile
constexpr int kKvStageWarps = 8;
constexpr int kKvRowsPerWarp = 8;

// Two e4m3 codes (low byte first) -> two floats, exactly.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
    return __half22float2(*reinterpret_cast<__half2*>(&h2));
}

// Dequantizes one 16-code chunk (tile scale s) into 16 bf16 values at dst.
__device__ __forceinline__ void stage_chunk(uint4 raw, float s, uint4* dst) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 lo = e4m3x2_to_float2((uint16_t)(w[k] & 0xFFFFu));
        const float2 hi = e4m3x2_to_float2((uint16_t)(w[k] >> 16));
        const __nv_bfloat162 a = __floats2bfloat162_rn(lo.x * s, lo.y * s);
        const __nv_bfloat162 b = __floats2bfloat162_rn(hi.x * s, hi.y * s);
        o[2 * k] = *reinterpret_cast<const uint32_t*>(&a);
        o[2 * k + 1] = *reinterpret_cast<const uint32_t*>(&b);
    }
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

// grid (ceil(K / 64), tc), 256 threads.  Each warp takes 8 consecutive selected
// rows of one token: lane l < 8 resolves row j0 + l (index, page, cache row), then
// every load of the 8 rows is issued before any conversion, so that a warp waits
// for one round of memory latency per row group.
__global__ void __launch_bounds__(32 * kKvStageWarps) kv_fp8_stage_kernel(const KvStageParams p) {
    // the attention launch that follows may be scheduled now (it waits for this grid
    // before reading anything written here)
    asm volatile("griddepcontrol.launch_dependents;" :::);
    const int i = blockIdx.y;                   // token of the chunk
    const int t = p.t0 + i;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pages = p.KP / kPage;
    __shared__ int s_b;
    if (threadIdx.x == 0) {
        int lo = 0, hi = p.B - 1;               // sequence of token t: last b with cu_q[b] <= t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldg(p.cu_q + mid) <= t) lo = mid;
            else hi = mid - 1;
        }
        s_b = lo;
    }
    if (blockIdx.x == 0) {
        for (int q = threadIdx.x; q < pages; q += blockDim.x) p.s_table[(int64_t)i * pages + q] = i * pages + q;
        if (threadIdx.x == 0) {
            p.s_seq_lens[i] = p.KP;
            p.s_cu_q[i] = i;
            if (i == p.tc - 1) p.s_cu_q[p.tc] = p.tc;
        }
    }
    __syncthreads();
    const int j0 = (blockIdx.x * kKvStageWarps + warp) * kKvRowsPerWarp;
    if (j0 >= p.K) return;
    const int j = j0 + lane;
    const bool mine = lane < kKvRowsPerWarp && j < p.K;
    const int pos = mine ? __ldg(p.idx + (int64_t)t * p.K + j) : -1;
    if (mine) p.s_idx[(int64_t)i * p.K + j] = pos >= 0 ? j : -1;
    long long row = -1;                          // cache row; -2: selected but out of range
    if (pos >= 0) {
        const int b = s_b;
        row = -2;
        if (pos < __ldg(p.seq_lens + b) && pos / kPage < p.max_blocks) {
            const int blk = __ldg(p.block_table + (int64_t)b * p.max_blocks + pos / kPage);
            if (blk >= 0 && blk < p.num_blocks) row = (long long)blk * kPage + pos % kPage;
        }
    }
    if (__any_sync(0xffffffffu, row == -2) && lane == 0) atomicCAS(p.status, 0u, (uint32_t)kStBounds);
    uint4* dst0 = reinterpret_cast<uint4*>(p.stage + ((int64_t)i * p.KP + j0) * kDqk);
    // 36 chunks of 16 codes per row: lane l takes chunk l and, for l < 4, chunk 32 + l;
    // chunk c lies in tile c / 8
    const int c1 = 32 + (lane & 3);
    constexpr int R = kKvRowsPerWarp;
    long long rr[R];
    uint4 a[R], b[R];
    float sa[R], sb[R];
#pragma unroll
    for (int u = 0; u < R; ++u) {
        rr[u] = __shfl_sync(0xffffffffu, row, u);
        if (rr[u] >= 0) {
            const uint4* src = reinterpret_cast<const uint4*>(p.kv_codes + rr[u] * kDqk);
            const float* sc = p.kv_scale + rr[u] * kKvTiles;
            a[u] = __ldg(src + lane);
            sa[u] = __ldg(sc + lane / 8);
            if (lane < 4) {
                b[u] = __ldg(src + c1);
                sb[u] = __ldg(sc + c1 / 8);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < R; ++u) {
        uint4* dst = dst0 + (int64_t)u * (kDqk / 8);
        if (rr[u] >= 0) {
            stage_chunk(a[u], sa[u], dst + 2 * lane);
            if (lane < 4) stage_chunk(b[u], sb[u], dst + 2 * c1);
        } else if (rr[u] == -2) {
            // a selected position past the cache: zeros (reported above)
            for (int c = lane; c < kDqk / 8; c += 32) dst[c] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

}  // namespace dsa
