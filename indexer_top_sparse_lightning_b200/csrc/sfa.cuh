// sfa.cuh -- split-K Sparse Flash Attention over selected MLA latent rows (sm_100a).
//
// The sparse read stage of the pages ("Day0 Adaptation and Sparse Attention
// Optimization for Long-Sequence LLM Inference", section 4: read the selected
// KV entries by blocks with vectorised indexed loads and compute attention
// only over them; "Optimizing and Deploying Ultra-Long Sequence Inference
// Architectures", section I).  For one query token with H <= 128 heads:
//
//   S = sm_scale * Q[128 x 576] . KV_sel[n x 576]^T,  P = softmax(S),
//   O = P . KV_sel[:, 0:512]
//
// Work split: a cluster of two CTAs owns one (token, row split).  O for 128
// heads x 512 dims in fp32 is exactly one SM's tensor memory, so the pair
// splits the 576-wide rows between them:
//   CTA 0 holds elements [0,256) and [512,576) of every row,
//   CTA 1 holds elements [256,512).
// Each CTA gathers only its bytes of each selected row (16-byte cp.async
// vector loads into 128-byte-swizzled shared memory), computes the partial
// logits S_c = Q_c . K_c^T on tcgen05 (M=128 heads, N=64 rows), and the two
// partial logit tiles are exchanged through distributed shared memory, so
// both CTAs hold the same full S (fp32 add is commutative, so both get the
// same bits) and make the same online-softmax decisions.  Each CTA then
// accumulates its 256-wide half of O = P . V in tensor memory (M=128, N=256,
// V read MN-major straight from the gathered rows).  No logit is computed
// twice and no row byte is fetched twice.
//
// Gather completion is signalled with cp.async.mbarrier.arrive.noinc, so each
// stage's barrier fires as soon as its own rows land.
// Roles per CTA: warps 0-3 softmax (thread h <-> head h <-> TMEM lane h),
// warps 4-7 row gather, warp 8 TMEM allocation and MMA issue.
// The running max uses a lazy rescale: O and l are rescaled only when the max
// grows by more than 2^8, otherwise the old reference max is kept.
// With several row splits per token, un-normalised partial O and (m, l) go to
// the workspace and a small combine kernel merges them.
#pragma once
#include "common.h"
#include "ptx.cuh"

namespace dsa {

struct SfaCfg {
    static constexpr int ROWS = 64;                     // selected rows per block
    static constexpr int NS = 2;                        // gather stages
    static constexpr int KBQ0 = 5, KBQ1 = 4;            // 64-wide K blocks held by CTA 0 / CTA 1
    static constexpr int KBMAX = 5;
    static constexpr int Q_BYTES = KBMAX * 128 * 128;   // [128 heads x 64] per K block
    static constexpr int KV_KB_BYTES = ROWS * 128;      // [64 rows x 64] per K block
    static constexpr int STAGE_BYTES = KBMAX * KV_KB_BYTES;
    static constexpr int P_BYTES = 128 * 128;           // [128 heads x 64 rows] bf16
    static constexpr int X_BYTES = 128 * ROWS * 4;      // peer's partial logits, fp32
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = OFF_Q + Q_BYTES;
    static constexpr int OFF_P = OFF_KV + NS * STAGE_BYTES;
    static constexpr int OFF_X = OFF_P + P_BYTES;
    static constexpr int OFF_MISC = OFF_X + X_BYTES;
    static constexpr int MISC_BYTES = 1024;
    static constexpr int MAX_ROWS = 2048;               // rows of one split (K <= 2048)
    static constexpr int OFF_ROWS = OFF_MISC + MISC_BYTES;
    static constexpr int OFF_VALID = OFF_ROWS + MAX_ROWS * 4;
    static constexpr int SMEM = 1024 + OFF_VALID + MAX_ROWS / 8;
    static constexpr int THREADS = 288;
    static constexpr int TMEM_COLS = 512;               // O: [0,256), S buffers: [256,320), [320,384)
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, ROWS, false, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 256, false, true);
};

struct SfaMisc {
    uint64_t q_full;
    uint64_t kv_full[SfaCfg::NS];
    uint64_t kv_empty[SfaCfg::NS];
    uint64_t s_full[2];
    uint64_t s_empty[2];
    uint64_t p_full;
    uint64_t p_empty;
    uint64_t o_full;
    uint64_t x_full;    // peer's partial logits have landed in my X buffer
    uint64_t x_free;    // peer has consumed the logits I wrote into its X buffer
    uint64_t drain;
    uint64_t rows_ready;   // physical rows and validity bits of the split are in shared memory
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ int token_sequence(const int32_t* cu_q, int B, int t) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu_q + mid) <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(SfaCfg::THREADS, 1)
    sfa_decode_kernel(const __grid_constant__ SfaParams p, const __grid_constant__ CUtensorMap tm_q) {
    using Cfg = SfaCfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* s_q = smem + Cfg::OFF_Q;
    uint8_t* s_kv = smem + Cfg::OFF_KV;
    uint8_t* s_p = smem + Cfg::OFF_P;
    float* s_x = reinterpret_cast<float*>(smem + Cfg::OFF_X);
    SfaMisc* m = reinterpret_cast<SfaMisc*>(smem + Cfg::OFF_MISC);
    int32_t* s_rows = reinterpret_cast<int32_t*>(smem + Cfg::OFF_ROWS);
    uint32_t* s_valid = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_VALID);
    volatile int* abort = &m->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = cluster_ctarank();
    const uint32_t peer = crank ^ 1u;
    const int cid = blockIdx.x >> 1;
    const int t = cid / p.n_splits;
    const int split = cid % p.n_splits;
    const int row_begin = split * p.rows_per_split;
    const int row_end = min(p.K, row_begin + p.rows_per_split);
    const int nblk = row_end > row_begin ? (row_end - row_begin + Cfg::ROWS - 1) / Cfg::ROWS : 0;
    const int kbq = crank == 0 ? Cfg::KBQ0 : Cfg::KBQ1;

    if (threadIdx.x == 0) {
        mbar_init(&m->q_full, 1);
        for (int i = 0; i < Cfg::NS; ++i) {
            mbar_init(&m->kv_full[i], 128);
            mbar_init(&m->kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&m->s_full[i], 1);
            mbar_init(&m->s_empty[i], 128);
        }
        mbar_init(&m->p_full, 128);
        mbar_init(&m->p_empty, 1);
        mbar_init(&m->o_full, 1);
        mbar_init(&m->x_full, 128);
        mbar_init(&m->x_free, 128);
        mbar_init(&m->drain, 1);
        mbar_init(&m->rows_ready, 128);
        m->abort = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(&m->tmem_base, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    if (p.H < 128) {
        // heads beyond H read zeros in the MMA (the Q loads bring exactly H rows)
        for (int i = threadIdx.x; i < Cfg::Q_BYTES / 16; i += blockDim.x)
            reinterpret_cast<uint4*>(s_q)[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    cluster_sync();   // barriers of both CTAs initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = m->tmem_base;
    const uint32_t tm_o = tmem_base;            // columns [0, 256)
    const uint32_t tm_s = tmem_base + 256;      // two 64-column logit buffers
    if (threadIdx.x == 0) DSA_TRACE_MARK(0);

    if (warp == 8) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            bool ok = true;
            // Q part of this CTA: K blocks at element offsets {0,64,128,192,512} or {256,...,448}
            mbar_arrive_expect_tx(&m->q_full, kbq * 64 * p.H * 2);
            for (int kb = 0; kb < kbq; ++kb) {
                const int x = crank == 0 ? (kb < 4 ? kb * 64 : 512) : 256 + kb * 64;
                tma_load_3d(s_q + kb * 128 * 128, &tm_q, &m->q_full, x, 0, t);
            }
            if (!mbar_wait(&m->q_full, 0, abort)) ok = false;
            tc_fence_after();
            const uint32_t q_addr = smem_u32(s_q);
            const uint32_t p_addr = smem_u32(s_p);
            auto issue_qk = [&](int jb) -> bool {
                const int s = jb % Cfg::NS, sb = jb & 1;
                if (!mbar_wait(&m->kv_full[s], (jb / Cfg::NS) & 1, abort)) return false;
                // rows were written by cp.async (generic proxy); the MMA reads them through the async proxy
                fence_proxy_async_smem();
                if (!mbar_wait(&m->s_empty[sb], ((jb >> 1) & 1) ^ 1, abort)) return false;
                tc_fence_after();
                const uint32_t kv_addr = smem_u32(s_kv + s * Cfg::STAGE_BYTES);
                for (int kb = 0; kb < kbq; ++kb)
                    for (int k16 = 0; k16 < 4; ++k16)
                        umma_bf16(tm_s + sb * Cfg::ROWS,
                                  sdesc_sw128(q_addr + kb * 16384 + k16 * 32, 16, 1024),
                                  sdesc_sw128(kv_addr + kb * Cfg::KV_KB_BYTES + k16 * 32, 16, 1024),
                                  Cfg::IDESC_QK, (kb | k16) != 0);
                umma_commit(&m->s_full[sb]);
                return true;
            };
            auto issue_pv = [&](int jb) -> bool {
                const int s = jb % Cfg::NS;
                if (!mbar_wait(&m->p_full, jb & 1, abort)) return false;
                tc_fence_after();
                const uint32_t kv_addr = smem_u32(s_kv + s * Cfg::STAGE_BYTES);
                for (int k16 = 0; k16 < 4; ++k16)
                    // A = P [128 heads x 64 rows] K-major; B = V [64 rows x 256 dims] MN-major:
                    // 64-dim groups are K blocks (LBO apart), 8-row groups 1024 B apart (SBO).
                    umma_bf16(tm_o, sdesc_sw128(p_addr + k16 * 32, 16, 1024),
                              sdesc_sw128(kv_addr + k16 * 16 * 128, Cfg::KV_KB_BYTES, 1024),
                              Cfg::IDESC_PV, (jb > 0 || k16 > 0));
                umma_commit(&m->kv_empty[s]);
                umma_commit(&m->p_empty);
                return true;
            };
            if (ok && nblk > 0) ok = issue_qk(0);
            for (int jb = 0; ok && jb < nblk; ++jb) {
                if (jb + 1 < nblk && !issue_qk(jb + 1)) { ok = false; break; }
                if (!issue_pv(jb)) { ok = false; break; }
            }
            umma_commit(&m->o_full);
            umma_commit(&m->drain);
            volatile int no_abort = 0;
            mbar_wait(&m->drain, 0, &no_abort);
            if (!ok) *abort = 1;
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- row gather
        const int pt = threadIdx.x - 128;           // 0..127
        const int b = token_sequence(p.cu_q, p.B, t);
        const int64_t L = __ldg(p.seq_lens + b);
        const int nch = kbq * 8;                    // 16-byte chunks per row held by this CTA
        const int32_t* idx_t = p.idx + (int64_t)t * p.K;
        const uint8_t* kv_bytes = reinterpret_cast<const uint8_t*>(p.kv);
        // physical row of every selected position of this split, and validity bits, once
        const int nrows = nblk * Cfg::ROWS;
        for (int i = pt; i < nrows; i += 128) {
            const int r = row_begin + i;
            int32_t row = -1;
            if (r < row_end) {
                const int32_t pos = __ldg(idx_t + r);
                if (pos >= 0) {
                    if (pos < L && pos / kPage < p.max_blocks) {
                        const int blk = __ldg(p.block_table + (int64_t)b * p.max_blocks + pos / kPage);
                        if (blk >= 0 && blk < p.num_blocks)
                            row = blk * kPage + pos % kPage;
                        else
                            atomicCAS(p.status, 0u, (uint32_t)kStBounds);
                    } else {
                        atomicCAS(p.status, 0u, (uint32_t)kStBounds);
                    }
                }
            }
            s_rows[i] = row;
            const uint32_t bits = __ballot_sync(0xffffffffu, row >= 0);
            if ((i & 31) == 0) s_valid[i >> 5] = bits;
        }
        mbar_arrive(&m->rows_ready);
        if (pt == 0) DSA_TRACE_MARK(1);
        named_bar_sync(2, 128);
        for (int jb = 0; jb < nblk; ++jb) {
            const int s = jb % Cfg::NS;
            if (!mbar_wait(&m->kv_empty[s], ((jb / Cfg::NS) & 1) ^ 1, abort)) break;
            const uint32_t st = smem_u32(s_kv + s * Cfg::STAGE_BYTES);
            const int32_t* rows = s_rows + jb * Cfg::ROWS;
            for (int e = pt; e < Cfg::ROWS * nch; e += 128) {
                const int r = e / nch, ch = e % nch;
                const int kb = ch >> 3, q = ch & 7;
                const int byte = crank == 0 ? (kb < 4 ? kb * 128 + q * 16 : 1024 + q * 16) : 512 + kb * 128 + q * 16;
                const int32_t row = rows[r];
                const void* src = kv_bytes + (row >= 0 ? (int64_t)row * (kDqk * 2) + byte : 0);
                cp_async_16(st + kb * Cfg::KV_KB_BYTES + r * 128 + ((q ^ (r & 7)) << 4), src, row >= 0);
            }
            // the barrier receives this thread's arrival once its copies have landed
            cp_async_arrive_noinc(&m->kv_full[s]);
        }
        cp_async_wait<0>();
    } else {
        // ---------------------------------------------------------------- softmax + epilogue
        const int h = threadIdx.x;                  // head == TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t x_full_peer = mapa_shared(smem_u32(&m->x_full), peer);
        const uint32_t x_free_peer = mapa_shared(smem_u32(&m->x_free), peer);
        const uint32_t x_peer_row = mapa_shared(smem_u32(s_x + h * Cfg::ROWS), peer);
        float mrun = -INFINITY, lrun = 0.0f;
        bool ok = nblk == 0 || mbar_wait(&m->rows_ready, 0, abort);
        for (int jb = 0; ok && jb < nblk; ++jb) {
            const int sb = jb & 1;
            // validity of the 64 rows of this block (same for every head)
            const uint32_t vmask[2] = {s_valid[jb * 2], s_valid[jb * 2 + 1]};
            if (!mbar_wait(&m->s_full[sb], (jb >> 1) & 1, abort)) { ok = false; break; }
            if (jb == 0 && h == 0) DSA_TRACE_MARK(2);
            tc_fence_after();
            uint32_t a[32], c[32];
            tmem_ld32(tm_s + lane_off + sb * Cfg::ROWS, a);
            tmem_ld32(tm_s + lane_off + sb * Cfg::ROWS + 32, c);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&m->s_empty[sb]);
            // exchange partial logits with the peer CTA
            if (!mbar_wait_cluster(&m->x_free, (jb & 1) ^ 1, abort)) { ok = false; break; }
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const uint32_t* src = q < 8 ? a : c;
                const int o = (q & 7) * 4;
                st_cluster_v4(x_peer_row + (uint32_t)(((q ^ (h & 15)) << 4)),
                              __uint_as_float(src[o]), __uint_as_float(src[o + 1]),
                              __uint_as_float(src[o + 2]), __uint_as_float(src[o + 3]));
            }
            mbar_arrive_remote(x_full_peer);
            if (!mbar_wait_cluster(&m->x_full, jb & 1, abort)) { ok = false; break; }
            float sv[64];
            const float* xrow = s_x + h * Cfg::ROWS;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float4 v = *reinterpret_cast<const float4*>(xrow + ((q ^ (h & 15)) << 2));
                const uint32_t* src = q < 8 ? a : c;
                const int o = (q & 7) * 4;
                sv[q * 4 + 0] = __uint_as_float(src[o + 0]) + v.x;
                sv[q * 4 + 1] = __uint_as_float(src[o + 1]) + v.y;
                sv[q * 4 + 2] = __uint_as_float(src[o + 2]) + v.z;
                sv[q * 4 + 3] = __uint_as_float(src[o + 3]) + v.w;
            }
            mbar_arrive_remote(x_free_peer);
            // online softmax in the log2 domain
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const bool v = (vmask[i >> 5] >> (i & 31)) & 1u;
                sv[i] = v ? sv[i] * p.scale_log2 : -INFINITY;
                mx = fmaxf(mx, sv[i]);
            }
            const float mnew = fmaxf(mrun, mx);
            const bool rescale = mnew > mrun + 8.0f;
            const float muse = rescale ? mnew : mrun;
            uint32_t pk[32];
            float rs = 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float p0 = muse == -INFINITY ? 0.0f : exp2f(sv[2 * i] - muse);
                const float p1 = muse == -INFINITY ? 0.0f : exp2f(sv[2 * i + 1] - muse);
                const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                const float2 pr = __bfloat1622float2(pb);
                rs += pr.x + pr.y;
                pk[i] = *reinterpret_cast<const uint32_t*>(&pb);
            }
            // P buffer free and O stable once the previous P.V has completed
            if (!mbar_wait(&m->p_empty, (jb & 1) ^ 1, abort)) { ok = false; break; }
            tc_fence_after();
            if (rescale && jb > 0) {
                const float f = exp2f(mrun - muse);
                lrun *= f;
#pragma unroll 1
                for (int c0 = 0; c0 < 256; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tm_o + lane_off + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                    tmem_st32(tm_o + lane_off + c0, o);
                }
                tmem_wait_st();
            }
            lrun += rs;
            mrun = muse;
            // P row h: 64 bf16 = 128 bytes, 128-byte swizzle
            uint8_t* prow = s_p + h * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<uint4*>(prow + ((q ^ (h & 7)) << 4)) =
                    make_uint4(pk[q * 4], pk[q * 4 + 1], pk[q * 4 + 2], pk[q * 4 + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&m->p_full);
        }
        // ---------------------------------------------------------------- epilogue
        if (h == 0) DSA_TRACE_MARK(3);
        if (ok && mbar_wait(&m->o_full, 0, abort)) {
            if (h == 0) DSA_TRACE_MARK(4);
            tc_fence_after();
            const int dim0 = crank == 0 ? 0 : 256;
            if (p.n_splits == 1) {
                const float inv = lrun > 0.0f ? 1.0f / lrun : 0.0f;
                for (int c0 = 0; c0 < 256; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tm_o + lane_off + c0, o);
                    tmem_wait_ld();
                    if (!(lrun > 0.0f))   // nothing selected: O was never written
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = 0u;
                    if (h < p.H) {
                        uint16_t* dst = p.out + ((int64_t)t * p.H + h) * kDv + dim0 + c0;
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            uint32_t w4[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[i + 2 * e]) * inv,
                                                                               __uint_as_float(o[i + 2 * e + 1]) * inv);
                                w4[e] = *reinterpret_cast<const uint32_t*>(&v);
                            }
                            *reinterpret_cast<uint4*>(dst + i) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                    }
                }
                if (crank == 0 && h < p.H && p.lse)
                    p.lse[(int64_t)t * p.H + h] = lrun > 0.0f ? (mrun + log2f(lrun)) * 0.69314718055994531f : -INFINITY;
            } else {
                // un-normalised partial: [t][split][dim chunk of 4][head][4]
                float* po = p.part_o + (((int64_t)t * p.n_splits + split) * 128) * 128 * 4;
                for (int c0 = 0; c0 < 256; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tm_o + lane_off + c0, o);
                    tmem_wait_ld();
                    if (!(lrun > 0.0f))
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = 0u;
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const int chunk = (dim0 + c0 + i) >> 2;
                        *reinterpret_cast<float4*>(po + ((int64_t)chunk * 128 + h) * 4) =
                            make_float4(__uint_as_float(o[i]), __uint_as_float(o[i + 1]),
                                        __uint_as_float(o[i + 2]), __uint_as_float(o[i + 3]));
                    }
                }
                if (crank == 0) {
                    float* ml = p.part_ml + ((int64_t)t * p.n_splits + split) * 256;
                    ml[h] = mrun;
                    ml[128 + h] = lrun;
                }
            }
        }
        if (!ok) *abort = 1;
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // no remote access may target an exited CTA
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
    if (threadIdx.x == 0 && m->abort) atomicCAS(p.status, 0u, (uint32_t)kStTimeout);
    if (threadIdx.x == 0) DSA_TRACE_MARK(9);
}

// Merge the row-split partials of each (token, head): weights 2^(m_s - M).
__global__ void __launch_bounds__(256) sfa_combine_kernel(const __grid_constant__ SfaParams p) {
    const int t = blockIdx.x / 64;
    const int sub = blockIdx.x % 64;
    const int pair = sub * 256 + threadIdx.x;      // (chunk, head) pair, 128 x 128
    const int chunk = pair / 128, h = pair % 128;
    const int S = p.n_splits;
    const float* ml = p.part_ml + (int64_t)t * S * 256;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, ml[s * 256 + h]);
    float Lsum = 0.0f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < S; ++s) {
        const float ms = ml[s * 256 + h];
        const float wgt = ms == -INFINITY ? 0.0f : exp2f(ms - M);
        Lsum += wgt * ml[s * 256 + 128 + h];
        const float4 v = *reinterpret_cast<const float4*>(
            p.part_o + ((((int64_t)t * S + s) * 128 + chunk) * 128 + h) * 4);
        acc.x += wgt * v.x;
        acc.y += wgt * v.y;
        acc.z += wgt * v.z;
        acc.w += wgt * v.w;
    }
    if (h >= p.H) return;
    const float inv = Lsum > 0.0f ? 1.0f / Lsum : 0.0f;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p.out + ((int64_t)t * p.H + h) * kDv + chunk * 4) = pk;
    if (chunk == 0 && p.lse)
        p.lse[(int64_t)t * p.H + h] = Lsum > 0.0f ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace dsa
