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

// Two e4m3 codes (low byte first) -> two floats, exactly.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
    return __half22float2(*reinterpret_cast<__half2*>(&h2));
}

// grid (ceil(KP / 8), tc), 256 threads: one warp per selected row of one token.
__global__ void __launch_bounds__(32 * kKvStageWarps) kv_fp8_stage_kernel(const KvStageParams p) {
    // the attention launch that follows may be scheduled now (it waits for this grid
    // before reading anything written here)
    asm volatile("griddepcontrol.launch_dependents;" :::);
    const int i = blockIdx.y;                   // token of the chunk
    const int t = p.t0 + i;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x * kKvStageWarps + warp;
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
    if (j >= p.K) return;
    const int pos = __ldg(p.idx + (int64_t)t * p.K + j);
    if (lane == 0) p.s_idx[(int64_t)i * p.K + j] = pos >= 0 ? j : -1;
    if (pos < 0) return;                        // never read by the attention
    const int b = s_b;
    int64_t row = -1;
    if (pos < __ldg(p.seq_lens + b) && pos / kPage < p.max_blocks) {
        const int blk = __ldg(p.block_table + (int64_t)b * p.max_blocks + pos / kPage);
        if (blk >= 0 && blk < p.num_blocks) row = (int64_t)blk * kPage + pos % kPage;
    }
    uint16_t* dst = p.stage + ((int64_t)i * p.KP + j) * kDqk;
    if (row < 0) {
        if (lane == 0) atomicCAS(p.status, 0u, (uint32_t)kStBounds);
        for (int c = lane; c < kDqk / 8; c += 32) reinterpret_cast<uint4*>(dst)[c] = make_uint4(0u, 0u, 0u, 0u);
        return;
    }
    const uint8_t* src = p.kv_codes + row * kDqk;
    const float* sc = p.kv_scale + row * kKvTiles;
    // 36 chunks of 16 codes; chunk c lies in tile c / 8
    for (int c = lane; c < kDqk / 16; c += 32) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src) + c);
        const float s = __ldg(sc + c / 8);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t o[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 lo = e4m3x2_to_float2((uint16_t)(w[k] & 0xFFFFu));
            const float2 hi = e4m3x2_to_float2((uint16_t)(w[k] >> 16));
            const __nv_bfloat162 a = __floats2bfloat162_rn(lo.x * s, lo.y * s);
            const __nv_bfloat162 bb = __floats2bfloat162_rn(hi.x * s, hi.y * s);
            o[2 * k] = *reinterpret_cast<const uint32_t*>(&a);
            o[2 * k + 1] = *reinterpret_cast<const uint32_t*>(&bb);
        }
        reinterpret_cast<uint4*>(dst)[2 * c] = make_uint4(o[0], o[1], o[2], o[3]);
        reinterpret_cast<uint4*>(dst)[2 * c + 1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

}  // namespace dsa
