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
// Work split: a cluster of two CTAs owns one (token, row split) and runs the
// two-CTA tensor-core MMA (tcgen05 cta_group::2, issued by CTA 0):
//   * CTA c holds Q for heads 64c..64c+63 (the A operand is split by M),
//   * per block of 32 selected rows, CTA c gathers rows 16c..16c+15 whole
//     (the B operand of S = Q.K^T is split by N), so each CTA receives the
//     full logits of its 64 heads over all 32 rows -- nothing is exchanged;
//   * for O = P.V, each CTA holds its own heads' P (A split by M) and the
//     value columns 128c..128c+127 and 256+128c..256+128c+127 of all 32 rows
//     (B split by N); each CTA's tensor memory receives O for its 64 heads
//     over all 512 columns.
// Rows are gathered with 16-byte asynchronous copies into the stages (one
// coalesced warp read per row segment; every free stage has its copies in
// flight) and written to 128-byte-swizzled shared memory;
// this CTA's own rows are prefetched into L2 a few blocks ahead.  The online
// softmax keeps a lazy reference max (O and l are rescaled only when the max
// grows by more than 2^8).  With several row splits per token, the last CTA of
// a (token, head half) to finish (arrival counted with a global atomic) merges
// the other splits' un-normalised partials and (m, l) into its own O, which
// never leaves tensor memory.
//
// Roles per CTA (512 threads): warps 0-3 softmax (thread L <-> TMEM lane L:
// head 64c + L%64, rows or value columns of half L/64), warps 4-14 gather,
// warp 15 TMEM allocation; in CTA 0 it issues the MMAs, in CTA 1 it forwards
// "my rows landed" and "my Q landed" to CTA 0.
#pragma once
#include "common.h"
#include "ptx.cuh"

namespace dsa {

struct SfaCfg {
    static constexpr int ROWS = 32;                     // selected rows per block (16 per CTA for S)
    static constexpr int NS = 4;                        // gather stages in shared memory
    static constexpr int NSB = 2;                       // logit / P buffers
    static constexpr int PF = 2;                        // blocks prefetched into L2 ahead of the gather
    static constexpr int KBQ = 9;                       // 64-wide K blocks of a 576-wide row
    static constexpr int Q_BYTES = KBQ * 64 * 128;      // [64 heads x 64] per K block
    static constexpr int KOWN_KB = 16 * 128;            // own 16 rows x 64 elements, per K block
    static constexpr int VALL_KB = ROWS * 128;          // all 32 rows x 64 value columns, per chunk
    static constexpr int STAGE_BYTES = KBQ * KOWN_KB + 4 * VALL_KB;
    static constexpr int P_BYTES = 64 * ROWS * 2;       // [64 heads x 32 rows] bf16, 64-byte rows
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = OFF_Q + Q_BYTES;
    static constexpr int OFF_P = OFF_KV + NS * STAGE_BYTES;
    static constexpr int OFF_MISC = OFF_P + NSB * P_BYTES;
    static constexpr int MISC_BYTES = 1024;
    static constexpr int MAX_ROWS = 2048;               // rows of one split (K <= 2048)
    static constexpr int OFF_ROWS = OFF_MISC + MISC_BYTES;
    static constexpr int OFF_XM = OFF_ROWS + MAX_ROWS * 4;    // partner max exchange [2][128]
    static constexpr int SMEM = 1024 + OFF_XM + 2 * 128 * 4;
    static constexpr int THREADS = 512;
    static constexpr int GATHER = 352;                  // threads of warps 4-14
    static constexpr int MMA_WARP = 15;                 // TMEM owner; MMA issuer (CTA 0) / forwarder (CTA 1)
    static constexpr int GATHER_ITEMS = 16 * 72 + 16 * 32;   // 16-byte loads of one block per CTA
    static constexpr int S_COLS = 16;                   // TMEM columns of one logit buffer
    static constexpr int TMEM_COLS = 512;               // O: [0,256), logit buffers from column 256
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, ROWS, false, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 256, false, true);
};

static_assert(SfaCfg::SMEM <= 227 * 1024, "attention shared memory exceeds the per-CTA limit");
static_assert(SfaCfg::MAX_ROWS / SfaCfg::ROWS <= 64, "the split merge keeps at most 64 splits");

struct SfaMisc {
    uint64_t q_full;            // own Q landed
    uint64_t q_peer;            // (CTA 0) the peer's Q landed
    uint64_t kv_full[SfaCfg::NS];
    uint64_t kv_peer[SfaCfg::NS];   // (CTA 0) the peer's rows of a stage landed
    uint64_t kv_empty[SfaCfg::NS];
    uint64_t s_full[SfaCfg::NSB];
    uint64_t s_empty[SfaCfg::NSB];  // (CTA 0) both CTAs read the logits
    uint64_t p_full[SfaCfg::NSB];   // (CTA 0) both CTAs wrote P
    uint64_t p_empty[SfaCfg::NSB];
    uint64_t o_full;
    uint64_t drain;
    uint64_t rows_ready;
    uint32_t tmem_base;
    int abort;
    int last;
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

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Arrive on an mbarrier of CTA 0 of the pair (a local arrive when this is CTA 0).
__device__ __forceinline__ void arrive_leader(uint64_t* bar, uint32_t crank) {
    if (crank == 0) mbar_arrive(bar);
    else mbar_arrive_remote(mapa_shared(smem_u32(bar), 0));
}

__global__ void __launch_bounds__(SfaCfg::THREADS, 1)
    sfa_decode_kernel(const __grid_constant__ SfaParams p, const __grid_constant__ CUtensorMap tm_q) {
    using Cfg = SfaCfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_shared(smem_raw, 1024);
    uint8_t* s_q = smem + Cfg::OFF_Q;
    uint8_t* s_kv = smem + Cfg::OFF_KV;
    uint8_t* s_p = smem + Cfg::OFF_P;
    SfaMisc* m = reinterpret_cast<SfaMisc*>(smem + Cfg::OFF_MISC);
    int32_t* s_rows = reinterpret_cast<int32_t*>(smem + Cfg::OFF_ROWS);
    float* s_xm = reinterpret_cast<float*>(smem + Cfg::OFF_XM);
    volatile int* abort = &m->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = cluster_ctarank();
    const int cid = blockIdx.x >> 1;
    const int t = cid / p.n_splits;
    const int split = cid % p.n_splits;
    const int row_begin = split * p.rows_per_split;
    const int row_end = min(p.K, row_begin + p.rows_per_split);
    const int nblk = row_end > row_begin ? (row_end - row_begin + Cfg::ROWS - 1) / Cfg::ROWS : 0;
    const int head0 = 64 * (int)crank;

    if (threadIdx.x == 0) {
        mbar_init(&m->q_full, 1);
        mbar_init(&m->q_peer, 1);
        for (int i = 0; i < Cfg::NS; ++i) {
            mbar_init(&m->kv_full[i], Cfg::GATHER);
            mbar_init(&m->kv_peer[i], 1);
            mbar_init(&m->kv_empty[i], 1);
        }
        for (int i = 0; i < Cfg::NSB; ++i) {
            mbar_init(&m->s_full[i], 1);
            mbar_init(&m->s_empty[i], 8);   // one arrival per softmax warp of both CTAs
            mbar_init(&m->p_full[i], 8);
            mbar_init(&m->p_empty[i], 1);
        }
        mbar_init(&m->o_full, 1);
        mbar_init(&m->drain, 1);
        mbar_init(&m->rows_ready, Cfg::GATHER);
        m->abort = 0;
        m->last = 0;
        fence_mbar_init();
    }
    if (warp == Cfg::MMA_WARP) {
        tmem_alloc_2cta(&m->tmem_base, Cfg::TMEM_COLS);
        tmem_relinquish_2cta();
    }
    if (p.H < 128) {
        // heads beyond H read zeros in the MMA (the Q loads bring only heads < H)
        for (int i = threadIdx.x; i < Cfg::Q_BYTES / 16; i += blockDim.x)
            reinterpret_cast<uint4*>(s_q)[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    cluster_sync();   // barriers of both CTAs initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = m->tmem_base;
    const uint32_t tm_o = tmem_base;            // columns [0, 256)
    const uint32_t tm_s = tmem_base + 256;      // logit buffers, S_COLS columns each
    if (threadIdx.x == 0) DSA_TRACE_MARK(0);

    if (warp == Cfg::MMA_WARP) {
        // ---------------------------------------------------------------- own Q
        if (lane == 0) {
            const int hb = p.H < 64 ? p.H : 64;              // TMA box height
            if (head0 < p.H) {
                mbar_arrive_expect_tx(&m->q_full, Cfg::KBQ * 64 * hb * 2);
                for (int kb = 0; kb < Cfg::KBQ; ++kb)
                    tma_load_3d(s_q + kb * 64 * 128, &tm_q, &m->q_full, kb * 64, head0, t);
            } else {
                mbar_arrive(&m->q_full);
            }
        }
        __syncwarp();
        volatile int no_abort = 0;
        if (crank == 1) {
            // ------------------------------------------------------------ forwarder
            if (lane == 0) {
                bool ok = mbar_wait(&m->q_full, 0, abort);
                if (ok) mbar_arrive_remote(mapa_shared(smem_u32(&m->q_peer), 0));
                for (int jb = 0; ok && jb < nblk; ++jb) {
                    const int s = jb % Cfg::NS;
                    if (!mbar_wait(&m->kv_full[s], (jb / Cfg::NS) & 1, abort)) { ok = false; break; }
                    DSA_TRACE_BLK(jb, 1);
                    // the rows were written by cp.async (generic proxy); CTA 0's MMA reads
                    // them through the async proxy
                    fence_proxy_async_smem();
                    mbar_arrive_remote(mapa_shared(smem_u32(&m->kv_peer[s]), 0));
                }
                if (!ok) *abort = 1;
            }
            __syncwarp();
        } else {
            // ------------------------------------------------------------ MMA issuer
            // The whole warp runs the schedule (decisions taken by lane 0 and
            // broadcast); one elected lane issues each group of MMAs and its commits.
            int q_ok = 0;
            if (lane == 0) q_ok = mbar_wait(&m->q_full, 0, abort) && mbar_wait(&m->q_peer, 0, abort);
            bool ok = __shfl_sync(0xffffffffu, q_ok, 0);
            tc_fence_after();
            const uint32_t q_addr = smem_u32(s_q);
            const uint32_t p_addr = smem_u32(s_p);
            auto qk_ready = [&](int jb) -> bool {
                const int s = jb % Cfg::NS, b = jb % Cfg::NSB;
                const uint32_t ph = (jb / Cfg::NS) & 1;
#ifdef DSA_TRACE
                const bool a = mbar_test_wait(smem_u32(&m->kv_full[s]), ph);
                const bool c = mbar_test_wait(smem_u32(&m->kv_peer[s]), ph);
                const bool e = mbar_test_wait(smem_u32(&m->s_empty[b]), ((jb / Cfg::NSB) & 1) ^ 1);
                if (a && g_dsa_trace_blk[jb & 63][12] == 0) DSA_TRACE_BLK(jb, 12);
                if (c && g_dsa_trace_blk[jb & 63][13] == 0) DSA_TRACE_BLK(jb, 13);
                if (e && g_dsa_trace_blk[jb & 63][14] == 0) DSA_TRACE_BLK(jb, 14);
                return a && c && e;
#else
                return mbar_test_wait(smem_u32(&m->kv_full[s]), ph) && mbar_test_wait(smem_u32(&m->kv_peer[s]), ph) &&
                       mbar_test_wait(smem_u32(&m->s_empty[b]), ((jb / Cfg::NSB) & 1) ^ 1);
#endif
            };
            auto pv_ready = [&](int jb) -> bool {
                return mbar_test_wait(smem_u32(&m->p_full[jb % Cfg::NSB]), (jb / Cfg::NSB) & 1);
            };
            auto issue_qk = [&](int jb) {
                const int s = jb % Cfg::NS, b = jb % Cfg::NSB;
                if (elect_one()) {
                    DSA_TRACE_BLK(jb, 6);
                    fence_proxy_async_smem();   // this CTA's cp.async rows -> async proxy
                    tc_fence_after();
                    const uint32_t kown = smem_u32(s_kv + s * Cfg::STAGE_BYTES);
#pragma unroll
                    for (int kb = 0; kb < Cfg::KBQ; ++kb)
#pragma unroll
                        for (int k16 = 0; k16 < 4; ++k16)
                            umma_bf16_2cta(tm_s + b * Cfg::S_COLS, sdesc_sw128(q_addr + kb * 8192 + k16 * 32, 16, 1024),
                                           sdesc_sw128(kown + kb * Cfg::KOWN_KB + k16 * 32, 16, 1024),
                                           Cfg::IDESC_QK, (kb | k16) != 0);
                    umma_commit_2cta(&m->s_full[b], 3);
                    DSA_TRACE_BLK(jb, 2);
                }
                __syncwarp();
            };
            auto issue_pv = [&](int jb) {
                const int s = jb % Cfg::NS, b = jb % Cfg::NSB;
                if (elect_one()) {
                    DSA_TRACE_BLK(jb, 7);
                    tc_fence_after();
                    const uint32_t vall = smem_u32(s_kv + s * Cfg::STAGE_BYTES + Cfg::KBQ * Cfg::KOWN_KB);
                    const uint32_t pb = p_addr + b * Cfg::P_BYTES;
#pragma unroll
                    for (int k16 = 0; k16 < 2; ++k16)
#pragma unroll
                        for (int half = 0; half < 2; ++half)  // value columns [256*half, 256*half+256)
                            // A = P [64 heads x 32 rows] K-major, 64-byte rows; B = V [32 rows x 128 columns
                            // per CTA] MN-major: 64-column chunks VALL_KB apart (LBO), 8-row groups 1024 B (SBO)
                            umma_bf16_2cta(tm_o + half * 128, sdesc_sw64(pb + k16 * 32, 16, 512),
                                           sdesc_sw128(vall + half * 2 * Cfg::VALL_KB + k16 * 16 * 128, Cfg::VALL_KB, 1024),
                                           Cfg::IDESC_PV, (jb > 0 || k16 > 0));
                    umma_commit_2cta(&m->kv_empty[s], 3);
                    umma_commit_2cta(&m->p_empty[b], 3);
                    DSA_TRACE_BLK(jb, 8);
                }
                __syncwarp();
            };
            int next_qk = 0, next_pv = 0;
            uint64_t t_idle = 0;
            while (ok && next_pv < nblk) {
                // P.V (four short MMAs that free a P buffer and a row stage) goes first
                // when a block's probabilities are ready; otherwise a block's logits go
                // ahead as soon as its rows and its logit buffer are free (the softmax of
                // block jb-NSB has read it), overlapping the softmax of earlier blocks
                // (lane 0 probes the barriers: 32 lanes probing one mbarrier serialise)
                int pv_ok = 0, qk_ok = 0;
                if (lane == 0) {
                    pv_ok = next_pv < next_qk && pv_ready(next_pv);
                    qk_ok = !pv_ok && next_qk < nblk && qk_ready(next_qk);
                }
                const bool do_pv = __shfl_sync(0xffffffffu, pv_ok, 0);
                const bool do_qk = __shfl_sync(0xffffffffu, qk_ok, 0);
                if (do_pv) {
                    issue_pv(next_pv++);
                    t_idle = 0;
                } else if (do_qk) {
                    issue_qk(next_qk++);
                    t_idle = 0;
                } else {
                    bool stop = *abort != 0;
                    const uint64_t now = globaltimer();
                    if (t_idle == 0) t_idle = now;
                    else if (now - t_idle > kWaitTimeoutNs) stop = true;
                    ok = !__shfl_sync(0xffffffffu, (int)stop, 0);
                }
            }
            if (elect_one()) {
                umma_commit_2cta(&m->o_full, 3);
                umma_commit_2cta(&m->drain, 1);
            }
            __syncwarp();
            mbar_wait(&m->drain, 0, &no_abort);
            if (!ok && lane == 0) *abort = 1;
        }
        // no TMA write may be in flight at exit
        if (lane == 0) mbar_wait(&m->q_full, 0, &no_abort);
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- row gather
        const int pt = threadIdx.x - 128;           // 0..GATHER-1
        const int gw = pt >> 5;                      // gather warp 0..10
        const int b = token_sequence(p.cu_q, p.B, t);
        const int64_t L = __ldg(p.seq_lens + b);
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
            }
        }
        mbar_arrive(&m->rows_ready);
        named_bar_sync(2, Cfg::GATHER);
        // The gather: every thread owns IPT fixed 16-byte items i = pt + GATHER*u of a
        // block and keeps the loads of one block in flight while it stores the
        // previous one.
        //   i < 1152        : own row i / 72, 16-byte chunk i % 72 (all 576 columns);
        //                     chunks of this CTA's value columns are stored twice
        //                     (logit operand and value operand)
        //   1152 <= i < 1664: peer row j / 32 (j = i - 1152), value chunk j % 32 of this
        //                     CTA's columns
        //   i >= 1664       : none (both bounds are multiples of 32: warp-uniform)
        // Skipped selections (row -1) load row 0; their logits are masked.
        constexpr int IPT = (Cfg::GATHER_ITEMS + Cfg::GATHER - 1) / Cfg::GATHER;
        constexpr int OWN_ITEMS = 16 * 72;
        static_assert(OWN_ITEMS % 32 == 0 && Cfg::GATHER_ITEMS % 32 == 0 && Cfg::GATHER % 32 == 0, "warp-uniform items");
        const int c = (int)crank;
        auto prefetch_block = [&](int jb) {
            if (gw == 0 && jb < nblk && lane < 16) {
                const int32_t row = s_rows[jb * Cfg::ROWS + 16 * c + lane];
                if (row >= 0) prefetch_l2(kv_bytes + (int64_t)row * (kDqk * 2), kDqk * 2);
            }
        };
        // Item descriptors are the same for every block: computed once.
        //   src[u]: byte offset in the row (bits 0-10), row of the block (bits 16-20);
        //           0xFFFFFFFF = no item
        //   dst[u]: stage offset of the logit or value copy (bits 0-15) and of the
        //           second (value) copy (bits 16-31, 0xFFFF = none)
        uint32_t src[IPT], dst[IPT];
#pragma unroll
        for (int u = 0; u < IPT; ++u) {
            const int i = pt + Cfg::GATHER * u;
            src[u] = 0xFFFFFFFFu;
            dst[u] = 0xFFFFFFFFu;
            if (i < OWN_ITEMS) {
                const int r = i / 72, ch = i % 72, kb = ch >> 3, q = ch & 7;
                const int sw = (q ^ (r & 7)) << 4;
                // value K blocks of this CTA: 2c, 2c+1 -> chunks 0, 1; 4+2c, 5+2c -> chunks 2, 3;
                // row 16c + r of a value chunk has the same swizzle phase as row r
                const int kr = kb - 2 * c;
                const int vq = (kr == 0 || kr == 1) ? kr : ((kr == 4 || kr == 5) ? kr - 2 : -1);
                src[u] = (uint32_t)(ch * 16) | ((uint32_t)(16 * c + r) << 16);
                const uint32_t d2 = vq >= 0 ? (uint32_t)(Cfg::KBQ * Cfg::KOWN_KB + vq * Cfg::VALL_KB + (16 * c + r) * 128 + sw)
                                            : 0xFFFFu;
                dst[u] = (uint32_t)(kb * Cfg::KOWN_KB + r * 128 + sw) | (d2 << 16);
            } else if (i < Cfg::GATHER_ITEMS) {
                const int j = i - OWN_ITEMS;
                const int v = j & 31, r = j >> 5;             // 8 chunks of each of 4 value K blocks
                const int kbv = v >> 3;
                const int kb = kbv < 2 ? 2 * c + kbv : 4 + 2 * c + (kbv - 2);
                src[u] = (uint32_t)(kb * 128 + (v & 7) * 16) | ((uint32_t)(16 * (1 - c) + r) << 16);
                dst[u] = (uint32_t)(Cfg::KBQ * Cfg::KOWN_KB + kbv * Cfg::VALL_KB + (16 * (1 - c) + r) * 128 +
                                    (((v & 7) ^ (r & 7)) << 4)) | (0xFFFFu << 16);
            }
        }
        static_assert(Cfg::STAGE_BYTES <= 0xFFFF, "stage offsets are packed in 16 bits");
        // one block: 16-byte asynchronous copies straight into the stage (own-row
        // value chunks copied twice), then this thread's arrival on the stage's
        // barrier once its copies have landed; a thread runs ahead as far as the
        // free stages allow
        auto issue = [&](int jb) -> bool {
            const int s = jb % Cfg::NS;
            if (!__all_sync(0xffffffffu, mbar_wait(&m->kv_empty[s], ((jb / Cfg::NS) & 1) ^ 1, abort))) return false;
            if (pt == 0) DSA_TRACE_BLK(jb, 5);
            const uint32_t base = smem_u32(s_kv + s * Cfg::STAGE_BYTES);
            const int32_t* rows = s_rows + jb * Cfg::ROWS;
#pragma unroll
            for (int u = 0; u < IPT; ++u) {
                if (src[u] == 0xFFFFFFFFu) continue;          // warp-uniform
                const int32_t r = rows[src[u] >> 16];
                const uint8_t* g = kv_bytes + (int64_t)(r < 0 ? 0 : r) * (kDqk * 2) + (src[u] & 0xFFFFu);
                cp_async_16(base + (dst[u] & 0xFFFFu), g, true);
                if ((dst[u] >> 16) != 0xFFFFu) cp_async_16(base + (dst[u] >> 16), g, true);
            }
            cp_async_arrive_noinc(&m->kv_full[s]);
            return true;
        };
        if (gw == 0 && lane == 0) DSA_TRACE_MARK(1);
        for (int jb = 0; jb < Cfg::PF; ++jb) prefetch_block(jb);
        bool ok = true;
        for (int jb = 0; ok && jb < nblk; ++jb) {
            prefetch_block(jb + Cfg::PF);
            ok = issue(jb);
        }
        cp_async_wait_all();
        if (!ok && lane == 0) *abort = 1;
    } else {
        // ---------------------------------------------------------------- softmax + epilogue
        const int L = threadIdx.x;                   // TMEM lane
        const int hl = L & 63;                       // local head
        const int half = L >> 6;                     // rows 16*half.. of a block; value columns of this half
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        float mrun = -INFINITY, lrun = 0.0f;
        // Every exit decision of these 128 threads is taken together (a vote
        // carried by the exchange barrier), so the named barriers always match.
        bool ok = nblk == 0 || mbar_wait(&m->rows_ready, 0, abort);
        for (int jb = 0; jb < nblk; ++jb) {
            const int b = jb % Cfg::NSB;
            // validity of this lane's 16 rows (skipped selections hold row -1)
            uint32_t vbits = 0;
            {
                const int4* r4 = reinterpret_cast<const int4*>(s_rows + jb * Cfg::ROWS + 16 * half);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int4 v = r4[q];
                    vbits |= (uint32_t)(v.x >= 0) << (4 * q) | (uint32_t)(v.y >= 0) << (4 * q + 1) |
                             (uint32_t)(v.z >= 0) << (4 * q + 2) | (uint32_t)(v.w >= 0) << (4 * q + 3);
                }
            }
            const bool got = __all_sync(0xffffffffu, ok && mbar_wait(&m->s_full[b], (jb / Cfg::NSB) & 1, abort));
            float sv[16];
            float mx0 = -INFINITY, mx1 = -INFINITY;
            if (got) {
                if (jb == 0 && L == 0) DSA_TRACE_MARK(2);
                if (L == 0) DSA_TRACE_BLK(jb, 0);
                tc_fence_after();
                uint32_t a[16];
                tmem_ld16(tm_s + lane_off + b * Cfg::S_COLS, a);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive_leader(&m->s_empty[b], crank);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float x = __uint_as_float(a[i]);
                    sv[i] = ((vbits >> i) & 1u) ? x * p.scale_log2 : -INFINITY;
                    if (i & 1) mx1 = fmaxf(mx1, sv[i]);
                    else mx0 = fmaxf(mx0, sv[i]);
                }
            }
            // the other 16 rows of this head are in lane L^64
            float* xm = s_xm + (jb & 1) * 128;
            xm[L] = fmaxf(mx0, mx1);
            ok = named_bar_and(1, 128, got);
            if (!ok) break;
            if (L == 0) DSA_TRACE_BLK(jb, 9);
            const float mx = fmaxf(xm[L], xm[L ^ 64]);
            const float mnew = fmaxf(mrun, mx);
            const bool rescale = mnew > mrun + 8.0f;      // identical in both lanes of a head
            const float muse = rescale ? mnew : mrun;
            const bool none = muse == -INFINITY;
            uint32_t pk[8];
            float rs0 = 0.0f, rs1 = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float p0 = none ? 0.0f : fast_exp2(sv[2 * i] - muse);
                const float p1 = none ? 0.0f : fast_exp2(sv[2 * i + 1] - muse);
                pk[i] = pack_bf16(p0, p1);
                // the row sum uses the bf16-rounded weights the MMA multiplies with
                rs0 += __uint_as_float(pk[i] << 16);
                rs1 += __uint_as_float(pk[i] & 0xFFFF0000u);
            }
            if (L == 0) DSA_TRACE_BLK(jb, 10);
            // P buffer b is free once P.V of block jb-NSB completed
            if (!__all_sync(0xffffffffu, mbar_wait(&m->p_empty[b], ((jb / Cfg::NSB) & 1) ^ 1, abort))) {
                ok = false;
                *abort = 1;
                continue;
            }
            if (L == 0) DSA_TRACE_BLK(jb, 3);
            const bool need = rescale && jb > 0;
            if (__any_sync(0xffffffffu, need)) {
                // O must be stable: P.V of block jb-1 has completed.  TMEM loads and
                // stores are warp-wide: lanes whose head keeps its max scale by 1.
                const int pb = (jb - 1) % Cfg::NSB;
                if (!__all_sync(0xffffffffu, mbar_wait(&m->p_empty[pb], ((jb - 1) / Cfg::NSB) & 1, abort))) {
                    ok = false;
                    *abort = 1;
                    continue;
                }
                tc_fence_after();
                const float f = need ? fast_exp2(mrun - muse) : 1.0f;
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
            lrun += rs0 + rs1;
            mrun = muse;
            // P row hl, 16 rows of this half: two 16-byte chunks of the 64-byte row (64-byte swizzle)
            uint8_t* prow = s_p + b * Cfg::P_BYTES + hl * 64;
            const uint32_t sw = (uint32_t)((hl >> 1) & 3);
#pragma unroll
            for (int q = 0; q < 2; ++q)
                *reinterpret_cast<uint4*>(prow + (((uint32_t)(2 * half + q) ^ sw) << 4)) =
                    make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_leader(&m->p_full[b], crank);
            if (L == 0) DSA_TRACE_BLK(jb, 4);
        }
        // ---------------------------------------------------------------- epilogue
        if (L == 0) DSA_TRACE_MARK(3);
        // full row sum of the head: this lane's rows plus the partner lane's
        ok = named_bar_and(1, 128, ok);
        s_xm[L] = lrun;
        named_bar_sync(1, 128);
        const float ltot = lrun + s_xm[L ^ 64];
        const int head = head0 + hl;
        ok = named_bar_and(1, 128, ok && mbar_wait(&m->o_full, 0, abort));
        if (ok) {
            if (L == 0) DSA_TRACE_MARK(4);
            tc_fence_after();
            const bool empty = !(ltot > 0.0f);   // nothing selected: O was never written
            if (p.n_splits == 1) {
                const float inv = empty ? 0.0f : 1.0f / ltot;
                for (int c0 = 0; c0 < 256; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tm_o + lane_off + c0, o);
                    tmem_wait_ld();
                    // columns 0-127: value columns 128*half + c; 128-255: 256 + 128*half + c
                    const int col = (c0 < 128 ? 128 * half + c0 : 256 + 128 * half + (c0 - 128));
                    if (head < p.H) {
                        uint16_t* dst = p.out + ((int64_t)t * p.H + head) * kDv + col;
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = empty ? 0.f : __uint_as_float(o[i + e]) * inv;
                            *reinterpret_cast<uint4*>(dst + i) = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]),
                                                                            pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
                        }
                    }
                }
                if (half == 0 && head < p.H && p.lse)
                    p.lse[(int64_t)t * p.H + head] = empty ? -INFINITY : (mrun + log2f(ltot)) * 0.69314718055994531f;
            } else {
                // Several row splits: the arrival order picks the CTA that merges
                // (the last to arrive); it waits only for CTAs that arrived before
                // it, and those wait for nothing, so no residency assumption is made.
                const int S = p.n_splits;
                uint32_t* arrive = p.split_count + (int64_t)t * 2 + crank;
                uint32_t* ready = p.split_ready + (int64_t)t * 2 + crank;
                if (L == 0) m->last = atomicAdd(arrive, 1u) == (uint32_t)S - 1u;
                named_bar_sync(1, 128);
                // un-normalised partials [t][split][head half][512 columns][64 heads] and
                // their (m, l) [t][split][head half][64][2]: a warp stores 32 heads of one column
                auto part = [&](int sp) { return p.part_o + (((int64_t)t * S + sp) * 2 + crank) * (kDv * 64); };
                auto pml = [&](int sp) { return p.part_ml + (((int64_t)t * S + sp) * 2 + crank) * (64 * 2); };
                if (!m->last) {
                    float* dst = part(split);
                    for (int c0 = 0; c0 < 256; c0 += 32) {
                        uint32_t o[32];
                        tmem_ld32(tm_o + lane_off + c0, o);
                        tmem_wait_ld();
                        const int col = (c0 < 128 ? 128 * half + c0 : 256 + 128 * half + (c0 - 128));
#pragma unroll
                        for (int i = 0; i < 32; ++i) __stcg(dst + (col + i) * 64 + hl, empty ? 0.0f : __uint_as_float(o[i]));
                    }
                    if (half == 0) __stcg(reinterpret_cast<float2*>(pml(split)) + hl, make_float2(mrun, ltot));
                    __threadfence();
                    named_bar_sync(1, 128);
                    if (L == 0) atomicAdd(ready, 1u);
                } else {
                    if (L == 0) {
                        const uint64_t t0 = globaltimer();
                        while (ld_acquire_gpu(ready) < (uint32_t)S - 1u) {
                            if (globaltimer() - t0 > kWaitTimeoutNs) {
                                atomicCAS(p.status, 0u, (uint32_t)kStTimeout);
                                *abort = 1;
                                break;
                            }
                        }
                    }
                    named_bar_sync(1, 128);
                    if (!*abort) {
                        // weights 2^(m_s - M) per split (own split from registers), kept in the idle Q buffer
                        float* wts = reinterpret_cast<float*>(s_q);     // [S][128 threads]
                        float M = mrun;
                        for (int sp = 0; sp < S; ++sp)
                            if (sp != split) M = fmaxf(M, __ldcg(reinterpret_cast<const float2*>(pml(sp)) + hl).x);
                        float Lsum = 0.0f;
                        for (int sp = 0; sp < S; ++sp) {
                            const float2 v = sp == split ? make_float2(mrun, ltot)
                                                         : __ldcg(reinterpret_cast<const float2*>(pml(sp)) + hl);
                            const float w = (M == -INFINITY || v.x == -INFINITY) ? 0.0f : exp2f(v.x - M);
                            wts[sp * 128 + L] = w;
                            Lsum += w * v.y;
                        }
                        const float inv = Lsum > 0.0f ? 1.0f / Lsum : 0.0f;
                        for (int c0 = 0; c0 < 256; c0 += 32) {
                            uint32_t o[32];
                            tmem_ld32(tm_o + lane_off + c0, o);
                            tmem_wait_ld();
                            const int col = (c0 < 128 ? 128 * half + c0 : 256 + 128 * half + (c0 - 128));
                            // splits folded in index order whichever CTA merges: the result is
                            // the same bits on every call
                            float acc[32];
#pragma unroll
                            for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
                            for (int sp = 0; sp < S; ++sp) {
                                const float w = wts[sp * 128 + L];
                                if (w == 0.0f) continue;
                                if (sp == split) {
#pragma unroll
                                    for (int i = 0; i < 32; ++i) acc[i] = fmaf(w, __uint_as_float(o[i]), acc[i]);
                                } else {
                                    const float* src = part(sp) + col * 64 + hl;
#pragma unroll
                                    for (int i = 0; i < 32; ++i) acc[i] = fmaf(w, __ldcg(src + i * 64), acc[i]);
                                }
                            }
                            if (head < p.H) {
                                uint16_t* dst = p.out + ((int64_t)t * p.H + head) * kDv + col;
#pragma unroll
                                for (int i = 0; i < 32; i += 8)
                                    *reinterpret_cast<uint4*>(dst + i) =
                                        make_uint4(pack_bf16(acc[i] * inv, acc[i + 1] * inv), pack_bf16(acc[i + 2] * inv, acc[i + 3] * inv),
                                                   pack_bf16(acc[i + 4] * inv, acc[i + 5] * inv), pack_bf16(acc[i + 6] * inv, acc[i + 7] * inv));
                            }
                        }
                        if (half == 0 && head < p.H && p.lse)
                            p.lse[(int64_t)t * p.H + head] = Lsum > 0.0f ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
                        // every other split has arrived and signalled: ready for the next call
                        if (L == 0) {
                            *arrive = 0u;
                            *ready = 0u;
                        }
                    }
                }
            }
        }
        if (!ok) *abort = 1;
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // no remote access may target an exited CTA, and no MMA may read a freed tile
    if (warp == Cfg::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc_2cta(tmem_base, Cfg::TMEM_COLS);
    }
    if (threadIdx.x == 0 && m->abort) atomicCAS(p.status, 0u, (uint32_t)kStTimeout);
    if (threadIdx.x == 0) DSA_TRACE_MARK(9);
}

}  // namespace dsa
