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
// vector loads into 128-byte-swizzled shared memory, rows prefetched into L2
// two blocks ahead), computes the partial logits S_c = Q_c . K_c^T on
// tcgen05 (M=128 heads, N=64 rows), and the two partial logit tiles are
// exchanged through distributed shared memory, so both CTAs hold the same
// full S (fp32 add is commutative, so both get the same bits) and make the
// same online-softmax decisions.  Each CTA then accumulates its 256-wide half
// of O = P . V in tensor memory (M=128, N=256, V read MN-major straight from
// the gathered rows).  No logit is computed twice and no row byte is fetched
// twice.
//
// Roles per CTA: warps 0-3 softmax (thread h <-> head h <-> TMEM lane h),
// warps 4-6 row gather, warp 7 TMEM allocation and MMA issue.  The MMA warp
// issues whichever of the next logit tile and the pending P.V product is
// ready first.  The running max uses a lazy rescale: O and l are rescaled
// only when the max grows by more than 2^8.
// With several row splits per token, each CTA writes an un-normalised
// partial O and (m, l); the last CTA of a (token, half) to finish merges the
// partials of all splits (arrival counted with a global atomic), so no
// separate combine launch is needed.
#pragma once
#include "common.h"
#include "ptx.cuh"

namespace dsa {

struct SfaCfg {
    static constexpr int ROWS = 64;                     // selected rows per block
    static constexpr int NS = 2;                        // gather stages in shared memory
    static constexpr int PF = 2;                        // blocks prefetched into L2 ahead of the gather
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
    static constexpr int THREADS = 256;                   // 8 warps: the register file allows 255 per thread
    static constexpr int GATHER = 96;                   // threads of warps 4-6
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
    uint64_t x_full;       // peer's partial logits have landed in my X buffer
    uint64_t x_free;       // peer has consumed the logits I wrote into its X buffer
    uint64_t drain;
    uint64_t rows_ready;   // physical rows and validity bits of the split are in shared memory
    uint32_t tmem_base;
    int abort;
    int last;              // this CTA merges the split partials of its (token, half)
};

__device__ __forceinline__ int token_sequence(const int32_t* cu_q, int B, int t) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu_q + mid) <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
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
            mbar_init(&m->kv_full[i], Cfg::GATHER);
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
        mbar_init(&m->rows_ready, Cfg::GATHER);
        m->abort = 0;
        m->last = 0;
        fence_mbar_init();
    }
    if (warp == 7) {
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

    if (warp == 7) {
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
            // readiness of the two kinds of work, polled without blocking
            auto qk_ready = [&](int jb) -> bool {
                return mbar_try_wait(smem_u32(&m->kv_full[jb % Cfg::NS]), (jb / Cfg::NS) & 1) &&
                       mbar_try_wait(smem_u32(&m->s_empty[jb & 1]), ((jb >> 1) & 1) ^ 1);
            };
            auto pv_ready = [&](int jb) -> bool { return mbar_try_wait(smem_u32(&m->p_full), jb & 1); };
            auto issue_qk = [&](int jb) {
                const int s = jb % Cfg::NS, sb = jb & 1;
                DSA_TRACE_BLK(jb, 6);
                // rows were written by cp.async (generic proxy); the MMA reads them through the async proxy
                fence_proxy_async_smem();
                tc_fence_after();
                const uint32_t kv_addr = smem_u32(s_kv + s * Cfg::STAGE_BYTES);
                for (int kb = 0; kb < kbq; ++kb)
#pragma unroll
                    for (int k16 = 0; k16 < 4; ++k16)
                        umma_bf16(tm_s + sb * Cfg::ROWS,
                                  sdesc_sw128(q_addr + kb * 16384 + k16 * 32, 16, 1024),
                                  sdesc_sw128(kv_addr + kb * Cfg::KV_KB_BYTES + k16 * 32, 16, 1024),
                                  Cfg::IDESC_QK, (kb | k16) != 0);
                umma_commit(&m->s_full[sb]);
            };
            auto issue_pv = [&](int jb) {
                const int s = jb % Cfg::NS;
                DSA_TRACE_BLK(jb, 7);
                tc_fence_after();
                const uint32_t kv_addr = smem_u32(s_kv + s * Cfg::STAGE_BYTES);
#pragma unroll
                for (int k16 = 0; k16 < 4; ++k16)
                    // A = P [128 heads x 64 rows] K-major; B = V [64 rows x 256 dims] MN-major:
                    // 64-dim groups are K blocks (LBO apart), 8-row groups 1024 B apart (SBO).
                    umma_bf16(tm_o, sdesc_sw128(p_addr + k16 * 32, 16, 1024),
                              sdesc_sw128(kv_addr + k16 * 16 * 128, Cfg::KV_KB_BYTES, 1024),
                              Cfg::IDESC_PV, (jb > 0 || k16 > 0));
                umma_commit(&m->kv_empty[s]);
                umma_commit(&m->p_empty);
            };
            // QK(j) may run up to two blocks ahead of PV(j) (two logit buffers)
            int next_qk = 0, next_pv = 0;
            uint64_t t_idle = 0;
            while (ok && next_pv < nblk) {
                bool progressed = false;
                if (next_qk < nblk && next_qk <= next_pv + 1 && qk_ready(next_qk)) {
                    issue_qk(next_qk++);
                    progressed = true;
                } else if (next_pv < next_qk && pv_ready(next_pv)) {
                    issue_pv(next_pv++);
                    progressed = true;
                }
                if (progressed) {
                    t_idle = 0;
                } else if (*abort) {
                    ok = false;
                } else {
                    const uint64_t now = globaltimer();
                    if (t_idle == 0) t_idle = now;
                    else if (now - t_idle > kWaitTimeoutNs) ok = false;
                }
            }
            umma_commit(&m->o_full);
            umma_commit(&m->drain);
            volatile int no_abort = 0;
            mbar_wait(&m->drain, 0, &no_abort);
            if (!ok) *abort = 1;
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- row gather
        const int pt = threadIdx.x - 128;           // 0..GATHER-1
        const int b = token_sequence(p.cu_q, p.B, t);
        const int64_t L = __ldg(p.seq_lens + b);
        const int gw = pt >> 5;                      // gather warp 0..2
        const uint32_t lane_q = (uint32_t)(lane & 7);
        const uint32_t lane_kb_off = (uint32_t)(lane >> 3) * Cfg::KV_KB_BYTES;
        const int lane_byte = (crank == 0 ? 0 : 512) + lane * 16;
        const int32_t* idx_t = p.idx + (int64_t)t * p.K;
        const uint8_t* kv_bytes = reinterpret_cast<const uint8_t*>(p.kv);
        // physical row of every selected position of this split and its validity bit,
        // computed once with all loads of a thread in flight together
        const int nrows = nblk * Cfg::ROWS;
        constexpr int RPT = (Cfg::MAX_ROWS + Cfg::GATHER - 1) / Cfg::GATHER;
        int32_t pos[RPT], blk[RPT];
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const int i = pt + k * Cfg::GATHER;
            pos[k] = (i < nrows && row_begin + i < row_end) ? __ldg(idx_t + row_begin + i) : -1;
        }
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            blk[k] = -1;
            if (pos[k] >= 0) {
                if (pos[k] < L && pos[k] / kPage < p.max_blocks)
                    blk[k] = __ldg(p.block_table + (int64_t)b * p.max_blocks + pos[k] / kPage);
                else
                    atomicCAS(p.status, 0u, (uint32_t)kStBounds);
            }
        }
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const int i = pt + k * Cfg::GATHER;
            if (i < nrows) {                           // uniform per warp (nrows is a multiple of 32)
                int32_t row = -1;
                if (blk[k] >= 0 && blk[k] < p.num_blocks) row = blk[k] * kPage + pos[k] % kPage;
                else if (pos[k] >= 0 && blk[k] != -1) atomicCAS(p.status, 0u, (uint32_t)kStBounds);
                s_rows[i] = row;
                const uint32_t bits = __ballot_sync(0xffffffffu, row >= 0);
                if (lane == 0) s_valid[i >> 5] = bits;
            }
        }
        mbar_arrive(&m->rows_ready);
        if (pt == 0) DSA_TRACE_MARK(1);
        named_bar_sync(2, Cfg::GATHER);
        // L2 prefetch of the first blocks' rows (this CTA's part of each row)
        auto prefetch_block = [&](int jb) {
            if (jb < nblk && pt < Cfg::ROWS) {
                const int32_t row = s_rows[jb * Cfg::ROWS + pt];
                if (row >= 0) {
                    const uint8_t* r = kv_bytes + (int64_t)row * (kDqk * 2);
                    if (crank == 0) {
                        prefetch_l2(r, 512);
                        prefetch_l2(r + 1024, 128);
                    } else {
                        prefetch_l2(r + 512, 512);
                    }
                }
            }
        };
        for (int jb = 0; jb < Cfg::PF; ++jb) prefetch_block(jb);
        for (int jb = 0; jb < nblk; ++jb) {
            const int s = jb % Cfg::NS;
            prefetch_block(jb + Cfg::PF);
            if (!mbar_wait(&m->kv_empty[s], ((jb / Cfg::NS) & 1) ^ 1, abort)) break;
            if (pt == 0) DSA_TRACE_BLK(jb, 5);
            const uint32_t st = smem_u32(s_kv + s * Cfg::STAGE_BYTES);
            const int32_t* rows = s_rows + jb * Cfg::ROWS;
            // one warp per row: lane l copies 16 bytes of the row's 256 latent elements
            // (one coalesced 512-byte read), lanes 0-7 of CTA 0 also the 64 RoPE elements
            for (int r = gw; r < Cfg::ROWS; r += Cfg::GATHER / 32) {
                const int32_t row = rows[r];
                const bool ok_row = row >= 0;
                const uint8_t* src_row = kv_bytes + (ok_row ? (int64_t)row * (kDqk * 2) : 0);
                const uint32_t dst_row = st + r * 128;
                const uint32_t sw = (uint32_t)(r & 7);
                cp_async_16(dst_row + lane_kb_off + ((lane_q ^ sw) << 4), src_row + lane_byte, ok_row);
                if (crank == 0 && lane < 8)
                    cp_async_16(dst_row + 4 * Cfg::KV_KB_BYTES + ((lane_q ^ sw) << 4), src_row + 1024 + lane * 16, ok_row);
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
        const float* xrow = s_x + h * Cfg::ROWS;
        float mrun = -INFINITY, lrun = 0.0f;
        bool ok = nblk == 0 || mbar_wait(&m->rows_ready, 0, abort);
        for (int jb = 0; ok && jb < nblk; ++jb) {
            const int sb = jb & 1;
            // validity of the 64 rows of this block (same for every head)
            const uint32_t v0 = s_valid[jb * 2], v1 = s_valid[jb * 2 + 1];
            if (!mbar_wait(&m->s_full[sb], (jb >> 1) & 1, abort)) { ok = false; break; }
            if (jb == 0 && h == 0) DSA_TRACE_MARK(2);
            if (h == 0) DSA_TRACE_BLK(jb, 0);
            tc_fence_after();
            uint32_t a[32], c[32];
            tmem_ld32(tm_s + lane_off + sb * Cfg::ROWS, a);
            tmem_ld32(tm_s + lane_off + sb * Cfg::ROWS + 32, c);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&m->s_empty[sb]);
            // exchange partial logits with the peer CTA
            if (!mbar_wait_cluster(&m->x_free, (jb & 1) ^ 1, abort)) { ok = false; break; }
            if (h == 0) DSA_TRACE_BLK(jb, 1);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                st_cluster_v4(x_peer_row + (uint32_t)((q ^ (h & 15)) << 4), __uint_as_float(a[4 * q]),
                              __uint_as_float(a[4 * q + 1]), __uint_as_float(a[4 * q + 2]),
                              __uint_as_float(a[4 * q + 3]));
#pragma unroll
            for (int q = 0; q < 8; ++q)
                st_cluster_v4(x_peer_row + (uint32_t)(((q + 8) ^ (h & 15)) << 4), __uint_as_float(c[4 * q]),
                              __uint_as_float(c[4 * q + 1]), __uint_as_float(c[4 * q + 2]),
                              __uint_as_float(c[4 * q + 3]));
            mbar_arrive_remote(x_full_peer);
            if (h == 0) DSA_TRACE_BLK(jb, 8);
            if (!mbar_wait_cluster(&m->x_full, jb & 1, abort)) { ok = false; break; }
            if (h == 0) DSA_TRACE_BLK(jb, 2);
            float sv[64];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 v = *reinterpret_cast<const float4*>(xrow + ((q ^ (h & 15)) << 2));
                sv[4 * q + 0] = __uint_as_float(a[4 * q + 0]) + v.x;
                sv[4 * q + 1] = __uint_as_float(a[4 * q + 1]) + v.y;
                sv[4 * q + 2] = __uint_as_float(a[4 * q + 2]) + v.z;
                sv[4 * q + 3] = __uint_as_float(a[4 * q + 3]) + v.w;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 v = *reinterpret_cast<const float4*>(xrow + (((q + 8) ^ (h & 15)) << 2));
                sv[32 + 4 * q + 0] = __uint_as_float(c[4 * q + 0]) + v.x;
                sv[32 + 4 * q + 1] = __uint_as_float(c[4 * q + 1]) + v.y;
                sv[32 + 4 * q + 2] = __uint_as_float(c[4 * q + 2]) + v.z;
                sv[32 + 4 * q + 3] = __uint_as_float(c[4 * q + 3]) + v.w;
            }
            mbar_arrive_remote(x_free_peer);
            if (h == 0) DSA_TRACE_BLK(jb, 9);
            // online softmax in the log2 domain
            float mxs[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) mxs[u] = -INFINITY;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const uint32_t vw = i < 32 ? v0 : v1;
                sv[i] = ((vw >> (i & 31)) & 1u) ? sv[i] * p.scale_log2 : -INFINITY;
                mxs[i & 7] = fmaxf(mxs[i & 7], sv[i]);   // eight independent chains
            }
            const float mx = fmaxf(fmaxf(fmaxf(mxs[0], mxs[1]), fmaxf(mxs[2], mxs[3])),
                                   fmaxf(fmaxf(mxs[4], mxs[5]), fmaxf(mxs[6], mxs[7])));
            const float mnew = fmaxf(mrun, mx);
            const bool rescale = mnew > mrun + 8.0f;
            const float muse = rescale ? mnew : mrun;
            const bool none = muse == -INFINITY;
            uint32_t pk[32];
            float rss[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float p0 = none ? 0.0f : exp2f(sv[2 * i] - muse);
                const float p1 = none ? 0.0f : exp2f(sv[2 * i + 1] - muse);
                pk[i] = pack_bf16(p0, p1);
                // the row sum uses the bf16-rounded weights the MMA multiplies with
                rss[i & 3] += __uint_as_float(pk[i] << 16) + __uint_as_float(pk[i] & 0xFFFF0000u);
            }
            const float rs = (rss[0] + rss[1]) + (rss[2] + rss[3]);
            if (h == 0) DSA_TRACE_BLK(jb, 10);
            // P buffer free and O stable once the previous P.V has completed
            if (!mbar_wait(&m->p_empty, (jb & 1) ^ 1, abort)) { ok = false; break; }
            if (h == 0) DSA_TRACE_BLK(jb, 3);
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
            if (h == 0) DSA_TRACE_BLK(jb, 4);
        }
        // ---------------------------------------------------------------- epilogue
        if (h == 0) DSA_TRACE_MARK(3);
        if (ok && mbar_wait(&m->o_full, 0, abort)) {
            if (h == 0) DSA_TRACE_MARK(4);
            tc_fence_after();
            const int dim0 = crank == 0 ? 0 : 256;
            const bool empty = !(lrun > 0.0f);   // nothing selected: O was never written
            if (p.n_splits == 1) {
                const float inv = empty ? 0.0f : 1.0f / lrun;
                for (int c0 = 0; c0 < 256; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tm_o + lane_off + c0, o);
                    tmem_wait_ld();
                    if (h < p.H) {
                        uint16_t* dst = p.out + ((int64_t)t * p.H + h) * kDv + dim0 + c0;
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            const float f0 = empty ? 0.f : __uint_as_float(o[i]) * inv;
                            const float f1 = empty ? 0.f : __uint_as_float(o[i + 1]) * inv;
                            const float f2 = empty ? 0.f : __uint_as_float(o[i + 2]) * inv;
                            const float f3 = empty ? 0.f : __uint_as_float(o[i + 3]) * inv;
                            const float f4 = empty ? 0.f : __uint_as_float(o[i + 4]) * inv;
                            const float f5 = empty ? 0.f : __uint_as_float(o[i + 5]) * inv;
                            const float f6 = empty ? 0.f : __uint_as_float(o[i + 6]) * inv;
                            const float f7 = empty ? 0.f : __uint_as_float(o[i + 7]) * inv;
                            *reinterpret_cast<uint4*>(dst + i) =
                                make_uint4(pack_bf16(f0, f1), pack_bf16(f2, f3), pack_bf16(f4, f5), pack_bf16(f6, f7));
                        }
                    }
                }
                if (crank == 0 && h < p.H && p.lse)
                    p.lse[(int64_t)t * p.H + h] = empty ? -INFINITY : (mrun + log2f(lrun)) * 0.69314718055994531f;
            } else {
                // un-normalised partial: [t][split][dim chunk of 4][head][4]
                float* po = p.part_o + (((int64_t)t * p.n_splits + split) * 128) * 128 * 4;
                for (int c0 = 0; c0 < 256; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tm_o + lane_off + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const int chunk = (dim0 + c0 + i) >> 2;
                        float4 v = make_float4(__uint_as_float(o[i]), __uint_as_float(o[i + 1]),
                                               __uint_as_float(o[i + 2]), __uint_as_float(o[i + 3]));
                        if (empty) v = make_float4(0.f, 0.f, 0.f, 0.f);
                        *reinterpret_cast<float4*>(po + ((int64_t)chunk * 128 + h) * 4) = v;
                    }
                }
                // (m, l) of this split, one copy per half so each half's merger reads its own
                float* ml = p.part_ml + (((int64_t)t * p.n_splits + split) * 2 + crank) * 256;
                ml[h] = mrun;
                ml[128 + h] = lrun;
                // the last CTA of this (token, half) to get here merges all splits
                __threadfence();
                named_bar_sync(1, 128);
                if (h == 0) {
                    const uint32_t prev = atomicAdd(p.split_count + (int64_t)t * 2 + crank, 1u);
                    m->last = prev == (uint32_t)p.n_splits - 1u;
                }
                named_bar_sync(1, 128);
            }
        }
        if (!ok) *abort = 1;
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (p.n_splits > 1 && m->last && !m->abort) {
        // merge the splits of this (token, half): weights 2^(m_s - M) per head
        // (in the now idle exchange buffer), then every thread folds (head,
        // 4-dim chunk) pairs, loads coalesced across heads
        __threadfence();
        const int S = p.n_splits;
        const int dim0 = crank == 0 ? 0 : 256;
        float* wsm = s_x;                  // [S][128]
        float* linv = s_x + 32 * 128;      // [128]
        for (int h = threadIdx.x; h < 128; h += Cfg::THREADS) {
            float M = -INFINITY;
            for (int s = 0; s < S; ++s)
                M = fmaxf(M, __ldcg(p.part_ml + (((int64_t)t * S + s) * 2 + crank) * 256 + h));
            float Lsum = 0.0f;
            for (int s = 0; s < S; ++s) {
                const float* mls = p.part_ml + (((int64_t)t * S + s) * 2 + crank) * 256;
                const float ms = __ldcg(mls + h);
                const float w = ms == -INFINITY ? 0.0f : exp2f(ms - M);
                wsm[s * 128 + h] = w;
                Lsum += w * __ldcg(mls + 128 + h);
            }
            linv[h] = Lsum > 0.0f ? 1.0f / Lsum : 0.0f;
            if (crank == 0 && h < p.H && p.lse)
                p.lse[(int64_t)t * p.H + h] = Lsum > 0.0f ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < 128 * 64; e += Cfg::THREADS) {
            const int h = e & 127, chunk = (dim0 >> 2) + (e >> 7);
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s = 0; s < S; ++s) {
                const float ws = wsm[s * 128 + h];
                const float4 v = __ldcg(reinterpret_cast<const float4*>(
                    p.part_o + ((((int64_t)t * S + s) * 128 + chunk) * 128 + h) * 4));
                acc.x += ws * v.x;
                acc.y += ws * v.y;
                acc.z += ws * v.z;
                acc.w += ws * v.w;
            }
            const float inv = linv[h];
            if (h < p.H)
                *reinterpret_cast<uint2*>(p.out + ((int64_t)t * p.H + h) * kDv + chunk * 4) =
                    make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
        }
        if (threadIdx.x == 0) p.split_count[(int64_t)t * 2 + crank] = 0u;   // ready for the next call
    }
    cluster_sync();   // no remote access may target an exited CTA
    if (warp == 7) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
    if (threadIdx.x == 0 && m->abort) atomicCAS(p.status, 0u, (uint32_t)kStTimeout);
    if (threadIdx.x == 0) DSA_TRACE_MARK(9);
}

}  // namespace dsa
