// prolog.cuh -- the indexer prolog as one kernel: a tcgen05 GEMM of the
// stacked projection rows [W_q; W_k; W_w] against the step's hidden states,
// with the per-row epilogue fused in (query rounding or MXFP8 encoding, key
// RMS normalization and encoding into the paged key cache, head weights).
//
// The pages run the four prolog steps (query projection, key normalization,
// query quantization, head-weight projection) on two or three streams so that
// they overlap ("Day0 Adaptation and Performance Optimization for Novel
// Long-Sequence Reasoning Models", section 3; "Large Model Inference
// Acceleration ...", section 1.2).  Here the three projections are rows of one
// weight matrix, so they are one contraction, and normalization and encoding
// happen on the accumulators before anything reaches HBM: one launch, no
// intermediate tensors, nothing to overlap.
//
// Orientation: D^T[n, t] = sum_c W[n, c] * x[t, c].  The weight rows are the
// MMA's M side (128 per tile, TMEM lanes), the tokens its N side (BN per tile,
// TMEM columns), so that each epilogue thread owns one output row (two warps
// per TMEM lane quarter, each taking half of the token columns): an MXFP8 group
// (32 consecutive rows of one head) is one warp, and the key's RMS norm is a
// reduction over the warps holding the key rows.
//
// Work units are (row tile, token tile, K split).  With one split the unit's
// CTA runs the epilogue from TMEM.  With S splits (few tiles, e.g. decode)
// every split CTA stores its fp32 partial tile to the workspace and counts
// itself in; the last to arrive adds the S partials in split order (a fixed
// order, so results do not depend on timing) and runs the epilogue.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "common.h"
#include "ptx.cuh"

namespace dsa {

struct PrologParams {
    const float* gamma;          // [D_I] key normalization weight
    const int32_t* seq_lens;
    const int32_t* cu_q;
    const int32_t* block_table;
    uint16_t* q_bf16;            // [T, H_I*D_I] bf16 bits (bf16 queries), else null
    uint8_t* q_codes;            // [T, H_I*D_I] e4m3 codes (MXFP8 queries), else null
    uint8_t* q_scale;            // [T, H_I*D_I/32] shared exponents (MXFP8 queries)
    float* w_out;                // [T, H_I]
    uint16_t* k_bf16;            // key cache [num_blocks*64, D_I] bf16 bits (bf16 keys), else null
    uint8_t* k_codes;            // key cache [num_blocks*64, D_I] e4m3 codes (fp8 / MXFP8 keys), else null
    float* k_scale_f32;          // [num_blocks*64, D_I/64] (fp8 keys), else null
    uint8_t* k_scale_e8;         // [num_blocks*64, D_I/32] (MXFP8 keys), else null
    uint32_t* status;
    uint32_t* counters;          // [tiles] split arrivals (zero between launches)
    float* partials;             // [max(S, Sk)][tiles][BN][128] fp32 partial tiles (split tiles)
    int32_t T, H_I, D_I, HD, n_out;
    int32_t B, max_blocks, num_blocks;
    int32_t MT, NT, S, KB, units, group_m;
    int32_t mk, Sk;              // the row tile holding the key rows, and its split count
    int32_t evict_w;             // weights are read once: stream them with an evict-first hint
    int32_t w_packed;            // weights in the tile-packed layout (one 16 KB block per row tile and k-block)
    float eps;
};

struct PrologMisc {
    uint64_t full[8], empty[8], tfull[2], tempty[2], drain, pbar;
    uint32_t tmem_base;
    int abort;
    int last;
    int pad_;
    uint64_t wait_ns;
    float red_ss[2][2][4][8];    // key sum of squares per (column half, sub-chunk parity, lane quarter, column)
    float red_am[2][2][4][8];    // key amax, the same indexing, for the per-64 fp8 scale
    int64_t row[256];            // key-cache row of each token column (-1: none)
};

template <int BN>
struct PrologCfg {
    static_assert(BN == 32 || BN == 64 || BN == 128 || BN == 256, "token tile");
    static constexpr int THREADS = 320;             // 8 epilogue warps, TMA producer, MMA issuer
    static constexpr int EPI_THREADS = 256;         // two warps per TMEM lane quarter, each half the columns
    static constexpr int PRODUCER_WARP = 8;
    static constexpr int MMA_WARP = 9;
    static constexpr int A_BYTES = 128 * 128;       // 128 weight rows x 64 bf16, 128-byte swizzle
    static constexpr int B_BYTES = BN * 128;        // BN tokens x 64 bf16
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int NS = BN <= 64 ? 8 : (BN == 128 ? 6 : 4);
    static constexpr int TMEM_COLS = 2 * BN;        // two accumulator buffers
    static constexpr uint32_t IDESC = idesc_bf16_f32(128, BN, false, false);
    static constexpr int OFF_MISC = NS * STAGE_BYTES;
    static constexpr int SMEM = OFF_MISC + (int)sizeof(PrologMisc) + 1024;   // + alignment slack
};

__device__ __forceinline__ void prolog_status(uint32_t* status, uint32_t code) { atomicCAS(status, 0u, code); }

// Unit u -> (row tile, token tile, split, splits of that tile, k-block range).
// The row tile holding the key rows (mk) may be split more ways (Sk) than the
// others (S): its epilogue (RMS norm, scattered cache-row stores) is the
// longest, so in a single-wave plan its units stream fewer k-blocks and its
// epilogue overlaps the other tiles' streaming.  Its units come first; the
// others follow with their splits consecutive, in groups of group_m row tiles,
// token tile slowest inside a group, so that the CTAs running at one time
// share their weight and token tiles in L2.
__device__ __forceinline__ void prolog_unit(const PrologParams& p, int u, int& tile, int& mt, int& nt, int& ks,
                                            int& ns, int& kb0, int& kb1) {
    const int nk = p.NT * p.Sk;
    if (u < nk) {
        ns = p.Sk;
        ks = u % p.Sk;
        nt = u / p.Sk;
        mt = p.mk;
    } else {
        u -= nk;
        ns = p.S;
        ks = u % p.S;
        const int t = u / p.S;                // among the row tiles other than mk
        const int rows = p.MT - 1;
        const int per_group = p.group_m * p.NT;
        const int g = t / per_group;
        const int r = t - g * per_group;
        int gm = rows - g * p.group_m;
        if (gm > p.group_m) gm = p.group_m;
        mt = g * p.group_m + r % gm;
        if (mt >= p.mk) ++mt;
        nt = r / gm;
    }
    tile = mt * p.NT + nt;
    kb0 = (int)((int64_t)ks * p.KB / ns);
    kb1 = (int)((int64_t)(ks + 1) * p.KB / ns);
}

// Key-cache row of query token t: its position is seq_len - nq + (t - first
// token of its sequence); the page comes from the block table.  -1 when the
// batch description is inconsistent or the page id is out of range.
__device__ __forceinline__ int64_t prolog_cache_row(const PrologParams& p, int t) {
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {                       // last sequence whose first token is <= t
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(p.cu_q + mid) <= t) lo = mid;
        else hi = mid - 1;
    }
    const int q0 = __ldg(p.cu_q + lo);
    const int nq = __ldg(p.cu_q + lo + 1) - q0;
    if (t < q0 || t - q0 >= nq) return -1;
    const int64_t pos = (int64_t)__ldg(p.seq_lens + lo) - nq + (t - q0);
    if (pos < 0) return -1;
    const int64_t pg = pos / kPage;
    if (pg >= p.max_blocks) return -1;
    const int bid = __ldg(p.block_table + (int64_t)lo * p.max_blocks + pg);
    if (bid < 0 || bid >= p.num_blocks) return -1;
    return (int64_t)bid * kPage + pos % kPage;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// e4m3fn code of v: round to nearest even, saturated at +-448 (the hardware
// conversion); a zero result is stored as +0.
__device__ __forceinline__ uint8_t e4m3_code(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(v));
    const uint8_t c = (uint8_t)(r & 0xFFu);
    return (c & 0x7Fu) ? c : (uint8_t)0;
}

// MX shared exponent of a group with largest magnitude amax: floor(log2 amax)
// minus 8 (the exponent of 256, the largest power of two in e4m3fn), clamped
// below at -127; an all-zero group takes 0 (scale 1).  Read off the fp32
// exponent field, so it is exact.
__device__ __forceinline__ int mx_exponent(float amax) {
    const int E = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
    if (E == 0) return amax > 0.0f ? -127 : 0;
    const int e = E - 127 - 8;
    return e < -127 ? -127 : e;
}
// 2^-e as fp32 for e in [-127, 119] (always a normal number).
__device__ __forceinline__ float mx_inv_scale(int e) { return __uint_as_float((uint32_t)(127 - e) << 23); }

template <int BN>
__global__ void __launch_bounds__(PrologCfg<BN>::THREADS, 1)
    indexer_prolog_kernel(const __grid_constant__ PrologParams p, const __grid_constant__ CUtensorMap tm_w,
                          const __grid_constant__ CUtensorMap tm_x) {
    using Cfg = PrologCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_shared(smem_raw, 1024);
    PrologMisc* m = reinterpret_cast<PrologMisc*>(smem + Cfg::OFF_MISC);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < Cfg::NS; ++i) {
            mbar_init(&m->full[i], 1);
            mbar_init(&m->empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&m->tfull[i], 1);
            mbar_init(&m->tempty[i], Cfg::EPI_THREADS);
        }
        mbar_init(&m->drain, 1);
        mbar_init(&m->pbar, 1);
        m->abort = 0;
        m->last = 0;
        // status area word 1: wait limit in microseconds (0: the default)
        const uint32_t us = __ldcg(p.status + 1);
        m->wait_ns = us ? (uint64_t)us * 1000u : kWaitTimeoutNs;
        fence_mbar_init();
    }
    if (warp == Cfg::MMA_WARP) {
        tmem_alloc(&m->tmem_base, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == Cfg::PRODUCER_WARP && lane == 0) {
        prefetch_tmap(&tm_w);
        prefetch_tmap(&tm_x);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = m->tmem_base;
    const uint64_t wlim = m->wait_ns;
    volatile int* abort = &m->abort;

    if (warp == Cfg::PRODUCER_WARP) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
                int tile, mt, nt, ks, ns, kb0, kb1;
                prolog_unit(p, u, tile, mt, nt, ks, ns, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % Cfg::NS;
                    if (!mbar_wait(&m->empty[s], ((it / Cfg::NS) & 1) ^ 1, abort, wlim)) { ok = false; break; }
                    uint8_t* st = smem + s * Cfg::STAGE_BYTES;
                    // rows or columns past the tensor's edge (last row tile, last token
                    // tile, a ragged last k-block) are filled with zeros by the copy
                    mbar_arrive_expect_tx(&m->full[s], Cfg::STAGE_BYTES);
                    if (p.w_packed) {
                        // block (mt, kb) of the packed weights: 16 KB contiguous
                        if (p.evict_w) tma_load_3d_hint(st, &tm_w, &m->full[s], 0, 0, mt * p.KB + kb, pol);
                        else tma_load_3d(st, &tm_w, &m->full[s], 0, 0, mt * p.KB + kb);
                    } else if (p.evict_w) {
                        tma_load_2d_hint(st, &tm_w, &m->full[s], kb * 64, mt * 128, pol);
                    } else {
                        tma_load_2d(st, &tm_w, &m->full[s], kb * 64, mt * 128);
                    }
                    tma_load_2d(st + Cfg::A_BYTES, &tm_x, &m->full[s], kb * 64, nt * BN);
                }
            }
            if (!ok) m->abort = 1;
            // drain: no copy may still be writing shared memory when the CTA exits
            const uint32_t first = it > (uint32_t)Cfg::NS ? it - Cfg::NS : 0u;
            volatile int no_abort = 0;
            for (uint32_t d = first; d < it; ++d)
                mbar_wait(&m->full[d % Cfg::NS], (d / Cfg::NS) & 1, &no_abort, wlim);
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t it = 0;
            int lu = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++lu) {
                int tile, mt, nt, ks, ns, kb0, kb1;
                prolog_unit(p, u, tile, mt, nt, ks, ns, kb0, kb1);
                const int buf = lu & 1;
                if (!mbar_wait(&m->tempty[buf], ((lu >> 1) & 1) ^ 1, abort, wlim)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + buf * BN;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % Cfg::NS;
                    if (!mbar_wait(&m->full[s], (it / Cfg::NS) & 1, abort, wlim)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * Cfg::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + Cfg::A_BYTES;
#pragma unroll
                    for (int k16 = 0; k16 < 4; ++k16) {
                        const uint64_t ad = sdesc_sw128(a_addr + k16 * 32, 16, 1024);
                        const uint64_t bd = sdesc_sw128(b_addr + k16 * 32, 16, 1024);
                        umma_bf16(d, ad, bd, Cfg::IDESC, (kb > kb0 || k16 > 0) ? 1u : 0u);
                    }
                    umma_commit(&m->empty[s]);
                }
                if (!ok) break;
                umma_commit(&m->tfull[buf]);
            }
            if (!ok) m->abort = 1;
            // drain: every issued MMA completes before TMEM is released
            umma_commit(&m->drain);
            volatile int no_abort = 0;
            mbar_wait(&m->drain, 0, &no_abort, wlim);
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 0-7)
        const int et = threadIdx.x;
        const int key_fp8_groups = p.k_scale_f32 != nullptr;
        int lu = 0;
        for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++lu) {
            int tile, mt, nt, ks, ns, kb0, kb1;
            prolog_unit(p, u, tile, mt, nt, ks, ns, kb0, kb1);
            const int buf = lu & 1;
            const int row0 = mt * 128;
            const int q4 = warp & 3;                     // TMEM lane quarter = the warp's 32 rows
            const int half = warp >> 2;                  // which half of the token columns
            const int cb = half * (BN / 2), ce = cb + BN / 2;
            const int base = row0 + q4 * 32;             // first output row of this warp
            const int n = base + lane;                   // this thread's output row
            const bool has_k = row0 < p.HD + p.D_I && row0 + 128 > p.HD;
            const bool kw = base >= p.HD && base < p.HD + p.D_I;   // this warp holds key rows
            named_bar_sync(1, Cfg::EPI_THREADS);        // every epilogue warp is done with the previous unit
            if (has_k) {
                for (int j = et; j < BN; j += Cfg::EPI_THREADS) {
                    const int t = nt * BN + j;
                    int64_t r = -1;
                    if (t < p.T) {
                        r = prolog_cache_row(p, t);
                        if (r < 0) prolog_status(p.status, kStBounds);
                    }
                    m->row[j] = r;
                }
            }
            const bool got = mbar_wait(&m->tfull[buf], (lu >> 1) & 1, abort, wlim);
            if (!named_bar_and(2, Cfg::EPI_THREADS, got)) {
                m->abort = 1;
                break;
            }
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(q4 * 32) << 16) + buf * BN;
            const int r_in = q4 * 32 + lane;
            bool fin = true;
            if (ns > 1) {
                // this split's partial tile, [BN columns][128 rows] fp32
                float* mine = p.partials + ((int64_t)ks * p.MT * p.NT + tile) * (BN * 128) + r_in;
#pragma unroll 1
                for (int c0 = cb; c0 < ce; c0 += 8) {
                    uint32_t r[8];
                    tmem_ld8(tb + c0, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 8; ++j) __stcg(mine + (c0 + j) * 128, __uint_as_float(r[j]));
                }
                __threadfence();
                named_bar_sync(3, Cfg::EPI_THREADS);
                if (et == 0) {
                    const uint32_t old = atomicAdd(p.counters + tile, 1u);
                    const int last = old == (uint32_t)(ns - 1);
                    if (last) p.counters[tile] = 0u;     // ready for the next launch
                    __threadfence();
                    m->last = last;
                }
                named_bar_sync(3, Cfg::EPI_THREADS);
                fin = m->last != 0;
            }
            if (fin && ns > 1) {
                // Add the S partials in split order into this CTA's accumulator (TMEM), then run
                // the epilogue from TMEM as for one split.  When every CTA has one unit (the
                // split plan makes it so) the stage ring is idle by now: the other splits'
                // tiles come in by bulk copies and are added from shared memory.  Otherwise
                // they are read from L2, four splits' loads in flight.
                const int64_t tsz = (int64_t)BN * 128;    // floats per partial tile
                const int64_t tiles = (int64_t)p.MT * p.NT;
                const bool staged = (int)gridDim.x >= p.units &&
                                    (ns - 1) * BN * 512 <= Cfg::NS * Cfg::STAGE_BYTES;
                const float* stg = reinterpret_cast<const float*>(smem);
                bool ok = true;
                if (staged) {
                    if (et == 0) {
                        fence_proxy_async_global();
                        mbar_arrive_expect_tx(&m->pbar, (uint32_t)((ns - 1) * BN * 512));
                        for (int s = 0, k = 0; s < ns; ++s) {
                            if (s == ks) continue;
                            bulk_load(smem + (int64_t)k * BN * 512, p.partials + ((int64_t)s * tiles + tile) * tsz,
                                      BN * 512, &m->pbar);
                            ++k;
                        }
                    }
                    ok = mbar_wait(&m->pbar, 0, abort, wlim);
                }
                if (!named_bar_and(2, Cfg::EPI_THREADS, ok)) {
                    m->abort = 1;
                    // no copy may still be writing shared memory when the CTA exits
                    if (et == 0) {
                        volatile int no_abort = 0;
                        mbar_wait(&m->pbar, 0, &no_abort, wlim);
                    }
                    break;
                }
#pragma unroll 1
                for (int c0 = cb; c0 < ce; c0 += 8) {
                    uint32_t r[8];
                    tmem_ld8(tb + c0, r);
                    tmem_wait_ld();
                    float v[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[j] = 0.0f;
                    if (staged) {
#pragma unroll 1
                        for (int s = 0; s < ns; ++s) {
                            if (s == ks) {
#pragma unroll
                                for (int j = 0; j < 8; ++j) v[j] += __uint_as_float(r[j]);
                            } else {
                                const float* ps = stg + (s - (s > ks ? 1 : 0)) * tsz + c0 * 128 + r_in;
#pragma unroll
                                for (int j = 0; j < 8; ++j) v[j] += ps[j * 128];
                            }
                        }
                    } else {
                        const float* part0 = p.partials + tile * tsz + c0 * 128 + r_in;
#pragma unroll 1
                        for (int s0 = 0; s0 < ns; s0 += 4) {
                            float a[4][8];
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const int s = s0 + q;
#pragma unroll
                                for (int j = 0; j < 8; ++j)
                                    a[q][j] = (s < ns && s != ks) ? __ldcg(part0 + s * tiles * tsz + j * 128)
                                                                   : __uint_as_float(r[j]);
                            }
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                if (s0 + q < ns)
#pragma unroll
                                    for (int j = 0; j < 8; ++j) v[j] += a[q][j];
                        }
                    }
                    uint32_t o[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) o[j] = __float_as_uint(v[j]);
                    tmem_st8(tb + c0, o);
                }
                tmem_wait_st();
            }
            if (fin) {
                // The epilogue walks the tile in sub-chunks of 8 token columns with rolled
                // loops: its code runs once per tile (the key tile on one CTA only), so it is
                // kept small enough to stay in the instruction cache.
                const int kw0 = (p.HD - row0) / 32;      // first warp holding key rows (has_k)
                const float g = kw ? __ldg(p.gamma + (base - p.HD) + lane) : 0.0f;
#pragma unroll 1
                for (int c0 = cb, cc = 0; c0 < ce; c0 += 8, ++cc) {
                    uint32_t r[8];
                    tmem_ld8(tb + c0, r);
                    tmem_wait_ld();
                    float v[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
                    const int t0 = nt * BN + c0;
                    const int rb = cc & 1;
                    if (has_k) {
                        // key rows: RMS normalization over the D_I rows of each token column
                        if (kw) {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const float s2 = warp_sum(v[j] * v[j]);
                                if (lane == 0) m->red_ss[half][rb][q4][j] = s2;
                            }
                        }
                        named_bar_sync(4, Cfg::EPI_THREADS);
                        if (kw) {
                            // lane j totals column j over the key warps (in warp order) and
                            // forms its factor; the factors are then broadcast
                            float fac = 0.0f;
                            if (lane < 8) {
                                float ss = 0.0f;
#pragma unroll
                                for (int w = 0; w < 4; ++w)
                                    if (w < p.D_I / 32) ss += m->red_ss[half][rb][kw0 + w][lane];
                                fac = rsqrtf(ss / (float)p.D_I + p.eps);
                            }
#pragma unroll
                            for (int j = 0; j < 8; ++j) v[j] = v[j] * __shfl_sync(0xffffffffu, fac, j) * g;
                        }
                        if (key_fp8_groups) {
                            if (kw) {
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const float a = warp_max(fabsf(v[j]));
                                    if (lane == 0) m->red_am[half][rb][q4][j] = a;
                                }
                            }
                            named_bar_sync(5, Cfg::EPI_THREADS);
                        }
                    }
                    if (base < p.HD) {
                        // ------------------------------------------------ queries
                        if (p.q_codes) {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int e = mx_exponent(warp_max(fabsf(v[j])));
                                const uint8_t c = e4m3_code(v[j] * mx_inv_scale(e));
                                const int t = t0 + j;
                                if (t < p.T) {
                                    p.q_codes[(int64_t)t * p.HD + n] = c;
                                    if (lane == 0) p.q_scale[(int64_t)t * (p.HD / 32) + base / 32] = (uint8_t)(e + 127);
                                }
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int t = t0 + j;
                                if (t < p.T) p.q_bf16[(int64_t)t * p.HD + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
                            }
                        }
                    } else if (kw) {
                        // ------------------------------------------------ keys into the paged cache
                        const int i = base - p.HD + lane;     // element of the key
                        const long long rowl = lane < 8 ? (long long)m->row[c0 + lane] : -1ll;
                        if (p.k_bf16) {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int64_t row = __shfl_sync(0xffffffffu, rowl, j);
                                if (row >= 0) p.k_bf16[row * p.D_I + i] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
                            }
                        } else if (key_fp8_groups) {
                            // the two warps of this 64-element scale group
                            const int w0 = kw0 + ((base - p.HD) / 64) * 2;
                            const bool first = ((base - p.HD) & 63) == 0;
                            float scl = 1.0f;
                            if (lane < 8) {
                                const float a = fmaxf(m->red_am[half][rb][w0][lane], m->red_am[half][rb][w0 + 1][lane]);
                                scl = a > 0.0f ? a / 448.0f : 1.0f;
                            }
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int64_t row = __shfl_sync(0xffffffffu, rowl, j);
                                const float sc = __shfl_sync(0xffffffffu, scl, j);
                                const uint8_t c = e4m3_code(v[j] / sc);
                                if (row >= 0) {
                                    p.k_codes[row * p.D_I + i] = c;
                                    if (lane == 0 && first) p.k_scale_f32[row * (p.D_I / 64) + (base - p.HD) / 64] = sc;
                                }
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int64_t row = __shfl_sync(0xffffffffu, rowl, j);
                                const int e = mx_exponent(warp_max(fabsf(v[j])));
                                const uint8_t c = e4m3_code(v[j] * mx_inv_scale(e));
                                if (row >= 0) {
                                    p.k_codes[row * p.D_I + i] = c;
                                    if (lane == 0) p.k_scale_e8[row * (p.D_I / 32) + (base - p.HD) / 32] = (uint8_t)(e + 127);
                                }
                            }
                        }
                    } else if (base >= p.HD + p.D_I && n < p.n_out) {
                        // ------------------------------------------------ head weights
                        const int h = n - p.HD - p.D_I;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int t = t0 + j;
                            if (t < p.T) p.w_out[(int64_t)t * p.H_I + h] = v[j];
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&m->tempty[buf]);
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == Cfg::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
    if (threadIdx.x == 0 && m->abort) prolog_status(p.status, kStTimeout);
}

// Tile-packed weight layout: block (mt, kb) -- rows 128*mt .. 128*mt+127 and
// columns 64*kb .. 64*kb+63 of the row-major [n_out, d] matrix, zero past its
// edges -- is stored row-major [128][64] at element offset (mt*KB + kb)*8192.
// One thread per 16-byte chunk of the packed array.
__global__ void __launch_bounds__(256) prolog_pack_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                          int n_out, int d, int KB, int64_t chunks) {
    for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < chunks; c += (int64_t)gridDim.x * blockDim.x) {
        const int c8 = (int)(c & 7);                  // 8 chunks of 8 elements per 64-column row
        const int r = (int)((c >> 3) & 127);
        const int64_t blk = c >> 10;
        const int kb = (int)(blk % KB);
        const int mt = (int)(blk / KB);
        const int row = mt * 128 + r;
        const int col = kb * 64 + c8 * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < n_out && col < d) v = src[((int64_t)row * d + col) / 8];   // d is a multiple of 8
        dst[c] = v;
    }
}

}  // namespace dsa
