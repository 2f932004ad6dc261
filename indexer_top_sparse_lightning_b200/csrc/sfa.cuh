// sfa.cuh -- Sparse Flash Attention over selected MLA latent rows (sm_100a).
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
// Work split.  The selected rows of all tokens form one list of 64-row blocks
// (token-major, ceil(K/64) blocks per token).  A cluster of two CTAs (one
// "pair") owns a contiguous range of that list: whole tokens when there are
// many more tokens than pairs, otherwise an even share of the list, so that
// every SM pair streams the same number of rows.  A token whose blocks are
// spread over several pairs gets one partial result per pair (normalised O in
// bf16 and the softmax statistics (m, l)), and a second, light kernel
// (sfa_combine_kernel, a programmatic dependent of this one) merges them.
//
// Per block the pair runs two-CTA tensor-core MMAs (tcgen05 cta_group::2,
// issued by CTA 0):
//   * S = Q.K^T with M = 128 heads (64 per CTA: A split by M) and N = 64 rows
//     (32 per CTA: B split by N): CTA c gathers block rows 32c..32c+31 whole
//     (all 576 columns) and receives the full logits of its 64 heads over all
//     64 rows -- no logit exchange;
//   * O += P.V with M = 128 heads and N = 256 value columns per MMA (two MMAs
//     cover the 512): CTA c holds value columns 128c.. and 256+128c.. of all
//     64 rows and its tensor memory receives O for its 64 heads over all 512.
// Selected rows arrive by TMA row gathers (tile::gather4: four rows of 64
// columns per instruction, written 128-byte swizzled straight into the MMA
// operand layout, completion counted in bytes on an mbarrier).  The copies
// bypass L1, whose share of the unified on-chip memory is small next to the
// 227 KB of stages, so the bytes in flight are bounded by the stages alone.
// One warp issues a row gather only every ~100 cycles per lane, so the
// gathers of a stage are spread over six warps (the rate grows with the number
// of issuing warps, not of lanes).
// The logit part of a stage (own rows, all 576 columns) is refilled as soon as
// its QK has completed, the value part (this CTA's value columns of all 64
// rows) once its P.V has.  The online softmax keeps a lazy reference max (O
// and l are rescaled only when the max grows by more than 2^8).
//
// Roles per CTA (384 threads):
//   warps 0-3   softmax and epilogue (thread L <-> TMEM lane L: head 64c+L%64,
//               block rows 32*(L/64).. of the logits, value columns of half
//               L/64 of each 256-column MMA)
//   warp 4      TMEM allocation; CTA 0: MMA issuer; CTA 1: forwards "my rows
//               landed" and "my Q landed" to CTA 0
//   warp 5      row ids: selected position -> block table -> cache row, one
//               ring slot per block; loads Q of each token with TMA
//   warps 6-8   TMA row gathers of the logit part of each stage
//   warps 9-11  TMA row gathers of the value part of each stage
//
// The kernel is launched as a programmatic dependent of the launch before it:
// every thread waits for that launch with griddepcontrol.wait after its
// prologue (barriers, TMEM and, after the indexer, the first Q load), so the
// prologue overlaps the end of the indexer; all reads of the index list, the
// block table and the cache come after the wait.
#pragma once
#include "common.h"
#include "ptx.cuh"

namespace dsa {

struct SfaCfg {
    static constexpr int ROWS = 64;                     // selected rows per block
    static constexpr int HROWS = 32;                    // rows of a block gathered whole by one CTA
    static constexpr int NS = 2;                        // row stages (logit part and value part each)
    static constexpr int NSB = 2;                       // logit / P buffers
    static constexpr int NRB = 3;                       // row-id ring (blocks)
    static constexpr int KBQ = 9;                       // 64-wide K chunks of a 576-wide row
        static constexpr int Q_BYTES = KBQ * 64 * 128;      // [64 heads x 64] per chunk
    static constexpr int KOWN_KB = HROWS * 128;         // own 32 rows x 64 columns, per chunk
    static constexpr int VALL_KB = ROWS * 128;          // all 64 rows x 64 value columns, per chunk
    static constexpr int QK_STAGE = KBQ * KOWN_KB;      // 36864: own rows, all 576 columns
    static constexpr int V_STAGE = 4 * VALL_KB;         // 32768: all rows, this CTA's value columns
    static constexpr int P_BYTES = 64 * ROWS * 2;       // [64 heads x 64 rows] bf16, 128-byte rows
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_QK = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_QK + NS * QK_STAGE;
    static constexpr int OFF_P = OFF_V + NS * V_STAGE;
    static constexpr int OFF_ROWS = OFF_P + NSB * P_BYTES;
    static constexpr int OFF_XM = OFF_ROWS + NRB * ROWS * 4;     // partner max / sum exchange [128]
    static constexpr int OFF_MISC = OFF_XM + 128 * 4;
    static constexpr int MISC_BYTES = 768;
    static constexpr int SMEM = 1024 + OFF_MISC + MISC_BYTES;
    static constexpr int THREADS = 384;
    static constexpr int MMA_WARP = 4;
    static constexpr int ROW_WARP = 5;
    static constexpr int QK_WARP0 = 6;                  // warps 6-8: row gathers of the logit part
    static constexpr int V_WARP0 = 9;                   // warps 9-11: row gathers of the value part
    static constexpr int GATHER_WARPS = 3;              // issuing warps per part
    static constexpr int QK_OPS = (HROWS / 4) * KBQ;    // 72 four-row gathers per logit part
    static constexpr int V_OPS = (ROWS / 4) * 4;        // 64 four-row gathers per value part
    static constexpr int S_COLS = HROWS;                // TMEM columns of one logit buffer
    static constexpr int TMEM_COLS = 512;               // O: [0, 256), logit buffers from column 256
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, ROWS, false, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 256, false, true);
    // partial results of a token shared by several pairs, one slot per (pair, side, CTA):
    // normalised O in bf16 [64 heads][512] and (m, l) [64][2] fp32
    static constexpr int64_t SLOT_O = 64 * 512 * 2;
    static constexpr int64_t SLOT_BYTES = SLOT_O + 64 * 8;
    static constexpr int MAX_SPLITS = (kMaxTopK + ROWS - 1) / ROWS;   // a token meets at most this many pairs
    static constexpr int COMBINE_THREADS = 256;         // merge kernel: one warp per (token, head)
};

static_assert(SfaCfg::SMEM <= 232448, "attention shared memory exceeds the per-CTA limit");
static_assert(SfaCfg::OFF_QK % 1024 == 0 && SfaCfg::OFF_V % 1024 == 0 && SfaCfg::QK_STAGE % 1024 == 0 &&
                  SfaCfg::V_STAGE % 1024 == 0 && SfaCfg::OFF_P % 1024 == 0,
              "128-byte swizzled operands need 1024-byte alignment");
static_assert(SfaCfg::MAX_SPLITS <= 32, "the merge kernel keeps one split per lane");
static_assert(SfaCfg::QK_OPS <= 32 * SfaCfg::GATHER_WARPS && SfaCfg::V_OPS <= 32 * SfaCfg::GATHER_WARPS &&
                  SfaCfg::V_OPS >= SfaCfg::GATHER_WARPS,
              "one gather instruction per issuing warp and stage");

struct SfaMisc {
    uint64_t q_full;            // own Q landed
    uint64_t q_peer;            // (CTA 0) the peer's Q landed
    uint64_t q_empty;           // every QK of the current token completed (both CTAs)
    uint64_t qk_full[SfaCfg::NS];   // logit part of a stage landed
    uint64_t qk_peer[SfaCfg::NS];   // (CTA 0) the peer's logit part landed
    uint64_t qk_empty[SfaCfg::NS];  // the block's QK completed
    uint64_t v_full[SfaCfg::NS];    // value part of a stage landed
    uint64_t v_peer[SfaCfg::NS];    // (CTA 0) the peer's value part landed
    uint64_t v_empty[SfaCfg::NS];   // the block's P.V completed
    uint64_t s_full[SfaCfg::NSB];
    uint64_t s_empty[SfaCfg::NSB];  // (CTA 0) both CTAs read the logits
    uint64_t p_full[SfaCfg::NSB];   // (CTA 0) both CTAs wrote P
    uint64_t p_empty[SfaCfg::NSB];
    uint64_t o_full;
    uint64_t o_empty;           // (CTA 0) both CTAs' epilogues read O
    uint64_t drain;
    uint64_t rows_full[SfaCfg::NRB];
    uint64_t rows_empty[SfaCfg::NRB];
    uint32_t tmem_base;
    int abort;
    uint32_t inject;
    uint64_t wait_ns;
};
static_assert(sizeof(SfaMisc) <= SfaCfg::MISC_BYTES, "attention misc block exceeds its slot");

__device__ __forceinline__ int token_sequence(const int32_t* cu_q, int B, int t) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu_q + mid) <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
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

// The contiguous block range of pair `pr` among `np` pairs: [g0, g1) of `total`.
__device__ __forceinline__ int64_t pair_start(int64_t total, int pr, int np) { return total * pr / np; }
// The pair whose range holds global block g.
__device__ __forceinline__ int pair_of_block(int64_t total, int64_t g, int np) {
    return (int)(((g + 1) * np + total - 1) / total) - 1;
}

// Resolves block jj of the pair's range: token, first/last block of its segment.
struct SfaBlock {
    int t, lb;           // token, block index inside the token
    int seg;             // segment (token) index inside the pair's range
    bool first, last;    // first / last block of its segment
};
__device__ __forceinline__ SfaBlock sfa_block(int64_t g0, int64_t g1, int nb, int jj) {
    SfaBlock r;
    const int64_t g = g0 + jj;
    r.t = (int)(g / nb);
    r.lb = (int)(g % nb);
    r.seg = r.t - (int)(g0 / nb);
    r.first = jj == 0 || r.lb == 0;
    r.last = g + 1 == g1 || r.lb == nb - 1;
    return r;
}

__global__ void __launch_bounds__(SfaCfg::THREADS, 1)
    sfa_decode_kernel(const __grid_constant__ SfaParams p, const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_kv) {
    using Cfg = SfaCfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_shared(smem_raw, 1024);
    uint8_t* s_q = smem + Cfg::OFF_Q;
    uint8_t* s_qk = smem + Cfg::OFF_QK;
    uint8_t* s_v = smem + Cfg::OFF_V;
    uint8_t* s_p = smem + Cfg::OFF_P;
    int32_t* s_rows = reinterpret_cast<int32_t*>(smem + Cfg::OFF_ROWS);
    float* s_xm = reinterpret_cast<float*>(smem + Cfg::OFF_XM);
    SfaMisc* m = reinterpret_cast<SfaMisc*>(smem + Cfg::OFF_MISC);
    volatile int* abort = &m->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = cluster_ctarank();
    const int np = (int)(gridDim.x >> 1);
    const int pair = (int)(blockIdx.x >> 1);
    const int nb = (p.K + Cfg::ROWS - 1) / Cfg::ROWS;       // blocks per token
    const int64_t total = (int64_t)p.T * nb;
    // contiguous block ranges; with align_tokens they start at token boundaries
    const int64_t g0 = p.align_tokens ? (int64_t)nb * ((int64_t)p.T * pair / np) : pair_start(total, pair, np);
    const int64_t g1 = p.align_tokens ? (int64_t)nb * ((int64_t)p.T * (pair + 1) / np) : pair_start(total, pair + 1, np);
    const int nblk = (int)(g1 - g0);
    const int head0 = 64 * (int)crank;

    if (threadIdx.x == 0) {
        mbar_init(&m->q_full, 1);
        mbar_init(&m->q_peer, 1);
        mbar_init(&m->q_empty, 1);
        for (int i = 0; i < Cfg::NS; ++i) {
            mbar_init(&m->qk_full[i], Cfg::GATHER_WARPS);   // one byte-counted arrival per issuing warp
            mbar_init(&m->qk_peer[i], 1);
            mbar_init(&m->qk_empty[i], 1);
            mbar_init(&m->v_full[i], Cfg::GATHER_WARPS);
            mbar_init(&m->v_peer[i], 1);
            mbar_init(&m->v_empty[i], 1);
        }
        for (int i = 0; i < Cfg::NSB; ++i) {
            mbar_init(&m->s_full[i], 1);
            mbar_init(&m->s_empty[i], 8);   // one arrival per softmax warp of both CTAs
            mbar_init(&m->p_full[i], 8);
            mbar_init(&m->p_empty[i], 1);
        }
        mbar_init(&m->o_full, 1);
        mbar_init(&m->o_empty, 8);
        mbar_init(&m->drain, 1);
        for (int i = 0; i < Cfg::NRB; ++i) {
            mbar_init(&m->rows_full[i], 1);
            mbar_init(&m->rows_empty[i], 4 + 2 * Cfg::GATHER_WARPS);   // softmax and gather warps
        }
        m->abort = 0;
        // test hooks in the status area: word 1 = wait limit in microseconds
        // (0: the default), word 2 = fault injection bits
        const uint32_t us = __ldcg(p.status + 1);
        m->wait_ns = us ? (uint64_t)us * 1000u : kWaitTimeoutNs;
        m->inject = __ldcg(p.status + 2);
        fence_mbar_init();
    }
    if (warp == Cfg::MMA_WARP) {
        tmem_alloc_2cta(&m->tmem_base, Cfg::TMEM_COLS);
        tmem_relinquish_2cta();
    }
    if (warp == Cfg::ROW_WARP && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_kv);
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
    const uint64_t wlim = m->wait_ns;
    const uint32_t inject = m->inject;

    // the merge kernel (a programmatic dependent) may be scheduled on SMs this grid
    // leaves idle; it waits for the whole grid before reading the partials
    griddep_launch_dependents();
    // Q of the first token does not depend on the index list: when the preceding
    // launch is known not to write it, it is loaded before waiting
    if (!p.early_q) griddep_wait();
    auto load_q = [&](int t) {
        const int hb = p.H < 64 ? p.H : 64;
        if (head0 < p.H) {
            mbar_arrive_expect_tx(&m->q_full, Cfg::KBQ * 64 * hb * 2);
            for (int kb = 0; kb < Cfg::KBQ; ++kb) tma_load_3d(s_q + kb * 64 * 128, &tm_q, &m->q_full, kb * 64, head0, t);
        } else {
            mbar_arrive(&m->q_full);
        }
    };
    if (warp == Cfg::ROW_WARP && lane == 0 && nblk > 0) load_q(sfa_block(g0, g1, nb, 0).t);
    // the index list is written by the preceding launch
    if (p.early_q) griddep_wait();

    if (warp == Cfg::MMA_WARP) {
        volatile int no_abort = 0;
        if (crank == 1) {
            // ------------------------------------------------------------ forwarder
            // One thread tells CTA 0 when this CTA's Q of a token, the logit part of a
            // stage and the value part of a stage have landed, whichever completes
            // first (the parts fill at different times).  The rows were written by
            // cp.async (generic proxy); CTA 0's MMA reads them through the async proxy.
            if (lane == 0) {
                int jq = 0, jk = 0, jv = 0;     // next block whose Q / logit part / value part to forward
                uint64_t t_idle = 0;
                bool ok = true;
                while (true) {
                    while (jq < nblk && !sfa_block(g0, g1, nb, jq).first) ++jq;
                    if (!ok || (jq >= nblk && jk >= nblk && jv >= nblk)) break;   // every Q forwarded too
                    bool moved = false;
                    if (jq < nblk && jq <= jk && mbar_test_wait(smem_u32(&m->q_full), sfa_block(g0, g1, nb, jq).seg & 1)) {
                        mbar_arrive_remote(mapa_shared(smem_u32(&m->q_peer), 0));
                        ++jq;
                        moved = true;
                    }
                    if (jk < nblk && mbar_test_wait(smem_u32(&m->qk_full[jk % Cfg::NS]), (jk / Cfg::NS) & 1)) {
                        fence_proxy_async_smem();
                        // test hook: CTA 0 never hears that this CTA's first rows landed
                        if (!(jk == 0 && (inject & 2u))) mbar_arrive_remote(mapa_shared(smem_u32(&m->qk_peer[jk % Cfg::NS]), 0));
                        ++jk;
                        moved = true;
                    }
                    if (jv < nblk && mbar_test_wait(smem_u32(&m->v_full[jv % Cfg::NS]), (jv / Cfg::NS) & 1)) {
                        fence_proxy_async_smem();
                        mbar_arrive_remote(mapa_shared(smem_u32(&m->v_peer[jv % Cfg::NS]), 0));
                        ++jv;
                        moved = true;
                    }
                    if (moved) {
                        t_idle = 0;
                    } else {
                        const uint64_t now = globaltimer();
                        if (*abort) ok = false;
                        else if (t_idle == 0) t_idle = now;
                        else if (now - t_idle > wlim) ok = false;
                    }
                }
                if (!ok) *abort = 1;
            }
            __syncwarp();
        } else {
            // ------------------------------------------------------------ MMA issuer
            // The whole warp runs the schedule (decisions by lane 0, broadcast); one
            // elected lane issues each group of MMAs and its commits.
            const uint32_t q_addr = smem_u32(s_q);
            const uint32_t p_addr = smem_u32(s_p);
            auto qk_ready = [&](int jj) -> bool {
                const SfaBlock bk = sfa_block(g0, g1, nb, jj);
                const int s = jj % Cfg::NS, b = jj % Cfg::NSB;
                const uint32_t ph = (jj / Cfg::NS) & 1;
                return mbar_test_wait(smem_u32(&m->q_full), bk.seg & 1) &&
                       mbar_test_wait(smem_u32(&m->q_peer), bk.seg & 1) && mbar_test_wait(smem_u32(&m->qk_full[s]), ph) &&
                       mbar_test_wait(smem_u32(&m->qk_peer[s]), ph) &&
                       mbar_test_wait(smem_u32(&m->s_empty[b]), ((jj / Cfg::NSB) & 1) ^ 1);
            };
            auto pv_ready = [&](int jj) -> bool {
                const SfaBlock bk = sfa_block(g0, g1, nb, jj);
                const int s = jj % Cfg::NS;
                const uint32_t ph = (jj / Cfg::NS) & 1;
                if (!mbar_test_wait(smem_u32(&m->p_full[jj % Cfg::NSB]), (jj / Cfg::NSB) & 1)) return false;
                if (!mbar_test_wait(smem_u32(&m->v_full[s]), ph) || !mbar_test_wait(smem_u32(&m->v_peer[s]), ph))
                    return false;
                // O of the previous token must have been read by both epilogues
                return !(bk.first && bk.seg > 0) || mbar_test_wait(smem_u32(&m->o_empty), (bk.seg - 1) & 1);
            };
            auto issue_qk = [&](int jj) {
                const SfaBlock bk = sfa_block(g0, g1, nb, jj);
                const int s = jj % Cfg::NS, b = jj % Cfg::NSB;
                if (elect_one()) {
                    fence_proxy_async_smem();   // this CTA's cp.async rows -> async proxy
                    tc_fence_after();
                    const uint32_t kown = smem_u32(s_qk + s * Cfg::QK_STAGE);
#pragma unroll
                    for (int kb = 0; kb < Cfg::KBQ; ++kb)
#pragma unroll
                        for (int k16 = 0; k16 < 4; ++k16)
                            umma_bf16_2cta(tm_s + b * Cfg::S_COLS, sdesc_sw128(q_addr + kb * 8192 + k16 * 32, 16, 1024),
                                           sdesc_sw128(kown + kb * Cfg::KOWN_KB + k16 * 32, 16, 1024),
                                           Cfg::IDESC_QK, (kb | k16) != 0);
                    umma_commit_2cta(&m->s_full[b], 3);
                    umma_commit_2cta(&m->qk_empty[s], 3);
                    if (bk.last) umma_commit_2cta(&m->q_empty, 3);   // Q may be replaced
                }
                __syncwarp();
            };
            auto issue_pv = [&](int jj) {
                const SfaBlock bk = sfa_block(g0, g1, nb, jj);
                const int s = jj % Cfg::NS, b = jj % Cfg::NSB;
                if (elect_one()) {
                    tc_fence_after();
                    const uint32_t vall = smem_u32(s_v + s * Cfg::V_STAGE);
                    const uint32_t pb = p_addr + b * Cfg::P_BYTES;
#pragma unroll
                    for (int k16 = 0; k16 < 4; ++k16)
#pragma unroll
                        for (int half = 0; half < 2; ++half)  // value columns [256*half, 256*half+256)
                            // A = P [64 heads x 64 rows] K-major, 128-byte rows; B = V [64 rows x 128
                            // columns per CTA] MN-major: 64-column chunks VALL_KB apart (LBO), 8-row
                            // groups 1024 B (SBO)
                            umma_bf16_2cta(tm_o + half * 128, sdesc_sw128(pb + k16 * 32, 16, 1024),
                                           sdesc_sw128(vall + half * 2 * Cfg::VALL_KB + k16 * 16 * 128, Cfg::VALL_KB, 1024),
                                           Cfg::IDESC_PV, (!bk.first || k16 > 0));
                    umma_commit_2cta(&m->v_empty[s], 3);
                    umma_commit_2cta(&m->p_empty[b], 3);
                    if (bk.last) umma_commit_2cta(&m->o_full, 3);
                }
                __syncwarp();
            };
            int next_qk = 0, next_pv = 0;
            uint64_t t_idle = 0;
            bool ok = true;
            while (ok && next_pv < nblk) {
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
                    else if (now - t_idle > wlim) stop = true;
                    ok = !__shfl_sync(0xffffffffu, (int)stop, 0);
                }
            }
            if (elect_one()) umma_commit_2cta(&m->drain, 1);
            __syncwarp();
            mbar_wait(&m->drain, 0, &no_abort, wlim);
            if (!ok && lane == 0) *abort = 1;
        }
    } else if (warp == Cfg::ROW_WARP) {
        // ---------------------------------------------------------------- row ids, Q loads
        // The warp runs up to NRB blocks ahead of the gathers.
        bool ok = true;
        int b = -1;
        int64_t L = 0;
        for (int jj = 0; ok && jj < nblk; ++jj) {
            const SfaBlock bk = sfa_block(g0, g1, nb, jj);
            const int r = jj % Cfg::NRB;
            if (!__all_sync(0xffffffffu, mbar_wait(&m->rows_empty[r], ((jj / Cfg::NRB) & 1) ^ 1, abort, wlim))) {
                ok = false;
                break;
            }
            if (bk.first) {
                b = token_sequence(p.cu_q, p.B, bk.t);
                L = __ldg(p.seq_lens + b);
            }
            const int32_t* idx_t = p.idx + (int64_t)bk.t * p.K;
            int32_t* ring = s_rows + r * Cfg::ROWS;
            int32_t rown[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = lane + 32 * h;
                const int k = bk.lb * Cfg::ROWS + i;
                rown[h] = k < p.K ? __ldg(idx_t + k) : -1;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int32_t pos = rown[h];
                int32_t row = -1;
                if (pos >= 0) {
                    if (pos < L && pos / kPage < p.max_blocks) {
                        const int blk = __ldg(p.block_table + (int64_t)b * p.max_blocks + pos / kPage);
                        if (blk >= 0 && blk < p.num_blocks) row = blk * kPage + pos % kPage;
                        else atomicCAS(p.status, 0u, (uint32_t)kStBounds);
                    } else {
                        atomicCAS(p.status, 0u, (uint32_t)kStBounds);
                    }
                }
                rown[h] = row;
                ring[lane + 32 * h] = row;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&m->rows_full[r]);
            // Q of a new token, once every QK of the previous one has completed (after
            // this block's rows are out: that QK needs the gathers they release)
            if (bk.first && jj > 0) {
                int qok = 1;
                if (lane == 0) {
                    qok = mbar_wait(&m->q_empty, (bk.seg - 1) & 1, abort, wlim);
                    if (qok) load_q(bk.t);
                }
                ok = __shfl_sync(0xffffffffu, qok, 0);
            }
        }
        if (!ok && lane == 0) *abort = 1;
        // no TMA write may be in flight at exit: the last Q load has landed
        if (lane == 0 && nblk > 0) {
            volatile int no_abort = 0;
            mbar_wait(&m->q_full, sfa_block(g0, g1, nb, nblk - 1).seg & 1, &no_abort, wlim);
        }
    } else if (warp >= Cfg::QK_WARP0 && warp < Cfg::V_WARP0 + Cfg::GATHER_WARPS) {
        // ---------------------------------------------------------------- TMA row gathers
        // Logit part (warps 6-8): own rows 32c..32c+31, all nine 64-column chunks, as 72
        // four-row gathers; value part (warps 9-11): this CTA's four value chunks of all 64
        // rows, 64 gathers.  Gather o of a part goes to lane o / 3 of issuing warp o % 3, so
        // each warp issues one instruction per stage (21 to 24 active lanes) and counts its
        // own bytes on the stage barrier.  Skipped selections (row -1) fetch row 0; their
        // logits are masked.
        const bool vpart = warp >= Cfg::V_WARP0;
        const int gw = warp - (vpart ? Cfg::V_WARP0 : Cfg::QK_WARP0);
        const int c = (int)crank;
        const int nops = vpart ? Cfg::V_OPS : Cfg::QK_OPS;
        const int o = lane * Cfg::GATHER_WARPS + gw;           // this lane's gather of the stage
        const int my_ops = (nops - gw + Cfg::GATHER_WARPS - 1) / Cfg::GATHER_WARPS;   // <= 32
        uint64_t* full = vpart ? m->v_full : m->qk_full;
        uint64_t* empty = vpart ? m->v_empty : m->qk_empty;
        uint8_t* stage0 = vpart ? s_v : s_qk;
        const int stage_bytes = vpart ? Cfg::V_STAGE : Cfg::QK_STAGE;
        // destination and source of gather o: logit part -- row group o / 9, chunk o % 9;
        // value part -- row group o / 4, value chunk slot o % 4
        int dst_off = 0, x = 0, g4 = 0;
        if (o < nops) {
            if (!vpart) {
                g4 = o / Cfg::KBQ;
                const int kb = o % Cfg::KBQ;
                dst_off = kb * Cfg::KOWN_KB + g4 * 512;
                x = kb * 64;
                g4 = 32 * c + 4 * g4;                          // first block row of the group
            } else {
                const int i = o >> 2, vch = o & 3;
                dst_off = vch * Cfg::VALL_KB + i * 512;
                x = (4 * (vch >> 1) + 2 * c + (vch & 1)) * 64;   // value chunk of the row
                g4 = 4 * i;
            }
        }
        bool ok = true;
        int issued = 0;
        for (int jj = 0; ok && jj < nblk; ++jj) {
            const int s = jj % Cfg::NS, r = jj % Cfg::NRB;
            if (!__all_sync(0xffffffffu, mbar_wait(&m->rows_full[r], (jj / Cfg::NRB) & 1, abort, wlim) &&
                                             mbar_wait(&empty[s], ((jj / Cfg::NS) & 1) ^ 1, abort, wlim))) {
                ok = false;
                break;
            }
            if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(my_ops * 512));
            __syncwarp();
            if (o < nops) {
                const int4 rr = *reinterpret_cast<const int4*>(s_rows + r * Cfg::ROWS + g4);
                tma_gather4(stage0 + s * stage_bytes + dst_off, &tm_kv, &full[s], x, rr.x < 0 ? 0 : rr.x,
                            rr.y < 0 ? 0 : rr.y, rr.z < 0 ? 0 : rr.z, rr.w < 0 ? 0 : rr.w);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&m->rows_empty[r]);
            issued = jj + 1;
        }
        if (!ok && lane == 0) *abort = 1;
        // no TMA write may be in flight at exit: the last stages issued have landed
        if (lane == 0) {
            volatile int no_abort = 0;
            for (int jd = issued > Cfg::NS ? issued - Cfg::NS : 0; jd < issued; ++jd)
                mbar_wait(&full[jd % Cfg::NS], (jd / Cfg::NS) & 1, &no_abort, wlim);
        }
    } else if (warp < 4) {
        // ---------------------------------------------------------------- softmax + epilogue
        const int L = threadIdx.x;                   // TMEM lane
        const int hl = L & 63;                       // local head
        const int half = L >> 6;                     // block rows 32*half..; value columns of this half
        const int head = head0 + hl;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        auto col_of = [&](int c0) { return c0 < 128 ? 128 * half + c0 : 256 + 128 * half + (c0 - 128); };
        // partial slot of split s_idx of token t (splits are the pairs pf.. in order): its
        // pair's first segment (side 0) unless that pair started in an earlier token
        auto slot = [&](int t, int pf, int s_idx) -> uint8_t* {
            const int pp = pf + s_idx;
            const int side = (s_idx == 0 && pair_start(total, pf, np) < (int64_t)t * nb) ? 1 : 0;
            return p.part + ((int64_t)(2 * pp + side) * 2 + crank) * Cfg::SLOT_BYTES;
        };
        float mrun = -INFINITY, lrun = 0.0f;
        bool ok = true;
        // Every exit decision of these 128 threads is taken together (votes carried
        // by named barriers), so the named barriers always match.
        for (int jj = 0; jj < nblk; ++jj) {
            const SfaBlock bk = sfa_block(g0, g1, nb, jj);
            const int b = jj % Cfg::NSB, r = jj % Cfg::NRB;
            if (bk.first) {
                mrun = -INFINITY;
                lrun = 0.0f;
            }
            // validity of this lane's 32 rows (skipped selections hold row -1)
            bool got = ok && mbar_wait(&m->rows_full[r], (jj / Cfg::NRB) & 1, abort, wlim);
            uint32_t vbits = 0;
            if (__all_sync(0xffffffffu, got)) {
                const int4* r4 = reinterpret_cast<const int4*>(s_rows + r * Cfg::ROWS + 32 * half);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int4 v = r4[q];
                    vbits |= (uint32_t)(v.x >= 0) << (4 * q) | (uint32_t)(v.y >= 0) << (4 * q + 1) |
                             (uint32_t)(v.z >= 0) << (4 * q + 2) | (uint32_t)(v.w >= 0) << (4 * q + 3);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&m->rows_empty[r]);
            }
            got = __all_sync(0xffffffffu, got && mbar_wait(&m->s_full[b], (jj / Cfg::NSB) & 1, abort, wlim));
            float sv[32];
            float mx = -INFINITY;
            if (got) {
                tc_fence_after();
                uint32_t a[32];
                tmem_ld32(tm_s + lane_off + b * Cfg::S_COLS, a);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive_leader(&m->s_empty[b], crank);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float x = __uint_as_float(a[i]);
                    sv[i] = ((vbits >> i) & 1u) ? x * p.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, sv[i]);
                }
            }
            // the other 32 rows of this head are in lane L^64 (one exchange slot: the
            // second vote below separates this read from the next block's write)
            s_xm[L] = mx;
            ok = named_bar_and(1, 128, got);
            if (!ok) break;
            const float mnew = fmaxf(mrun, fmaxf(mx, s_xm[L ^ 64]));
            const bool rescale = mnew > mrun + 8.0f;      // identical in both lanes of a head
            const float muse = rescale ? mnew : mrun;
            const bool none = muse == -INFINITY;
            uint32_t pk[16];
            float rs0 = 0.0f, rs1 = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float p0 = none ? 0.0f : fast_exp2(sv[2 * i] - muse);
                const float p1 = none ? 0.0f : fast_exp2(sv[2 * i + 1] - muse);
                pk[i] = pack_bf16(p0, p1);
                // the row sum uses the bf16-rounded weights the MMA multiplies with
                rs0 += __uint_as_float(pk[i] << 16);
                rs1 += __uint_as_float(pk[i] & 0xFFFF0000u);
            }
            // P buffer b is free once P.V of block jj-NSB completed
            if (!__all_sync(0xffffffffu, mbar_wait(&m->p_empty[b], ((jj / Cfg::NSB) & 1) ^ 1, abort, wlim))) {
                ok = false;
                *abort = 1;
            }
            const bool need = rescale && !bk.first;
            if (ok && __any_sync(0xffffffffu, need)) {
                // O must be stable: P.V of block jj-1 has completed.  TMEM loads and
                // stores are warp-wide: lanes whose head keeps its max scale by 1.
                const int pb = (jj - 1) % Cfg::NSB;
                if (!__all_sync(0xffffffffu, mbar_wait(&m->p_empty[pb], ((jj - 1) / Cfg::NSB) & 1, abort, wlim))) {
                    ok = false;
                    *abort = 1;
                } else {
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
            }
            // a failed wait above still reaches the vote below (the named barriers match)
            ok = named_bar_and(1, 128, ok);
            if (!ok) break;
            lrun += rs0 + rs1;
            mrun = muse;
            // P row hl, 32 rows of this half: four 16-byte chunks of the 128-byte row (128-byte swizzle)
            uint8_t* prow = s_p + b * Cfg::P_BYTES + hl * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4*>(prow + ((((uint32_t)(4 * half + q)) ^ (uint32_t)(hl & 7)) << 4)) =
                    make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_leader(&m->p_full[b], crank);

            if (!bk.last) continue;
            // ------------------------------------------------------------ epilogue of a token
            // full row sum of the head: this lane's rows plus the partner lane's
            s_xm[L] = lrun;
            const bool ofull = mbar_wait(&m->o_full, bk.seg & 1, abort, wlim);
            ok = named_bar_and(1, 128, ok && ofull);
            if (!ok) break;
            const float ltot = lrun + s_xm[L ^ 64];
            tc_fence_after();
            const bool empty = !(ltot > 0.0f);   // nothing selected: O was never written
            const int t = bk.t;
            const bool complete = g0 <= (int64_t)t * nb && g1 >= (int64_t)(t + 1) * nb;   // whole token here
            const float inv = empty ? 0.0f : 1.0f / ltot;
            if (complete) {
                for (int c0 = 0; c0 < 256; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tm_o + lane_off + c0, o);
                    tmem_wait_ld();
                    if (head < p.H) {
                        uint16_t* dstp = p.out + ((int64_t)t * p.H + head) * kDv + col_of(c0);
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(o[i + e]) * inv;
                            *reinterpret_cast<uint4*>(dstp + i) = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]),
                                                                             pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
                        }
                    }
                }
                if (half == 0 && head < p.H && p.lse)
                    p.lse[(int64_t)t * p.H + head] = empty ? -INFINITY : (mrun + log2f(ltot)) * 0.69314718055994531f;
            } else {
                // The token is shared with other pairs: this pair writes its normalised
                // partial O (bf16) and (m, l) to its slot; the merge kernel combines them.
                const int pf = pair_of_block(total, (int64_t)t * nb, np);
                uint8_t* sl = slot(t, pf, pair - pf);
                uint16_t* od = reinterpret_cast<uint16_t*>(sl) + hl * 512;
                for (int c0 = 0; c0 < 256; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tm_o + lane_off + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 8)
                        __stcg(reinterpret_cast<uint4*>(od + col_of(c0) + i),
                               make_uint4(pack_bf16(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv),
                                          pack_bf16(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv),
                                          pack_bf16(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv),
                                          pack_bf16(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv)));
                }
                if (half == 0)
                    __stcg(reinterpret_cast<float2*>(sl + Cfg::SLOT_O) + hl, make_float2(mrun, empty ? 0.0f : ltot));
            }
            // O has been read: the next token's first P.V may overwrite it
            tc_fence_before();
            named_bar_sync(1, 128);
            if (L % 32 == 0) arrive_leader(&m->o_empty, crank);
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
}

// Merge of the tokens whose blocks were spread over several pairs (the launcher
// starts it only when some token is).  One warp per (token, head): lane s reads
// the statistics (m_s, l_s) of split s (log2 units: m is the running maximum of
// the scaled logits, l the sum of 2^(logit - m) over the split's rows), the
// weights are 2^(m_s - M) * l_s with M the largest m_s, and each lane merges 16
// value columns of the splits' normalised outputs in split order:
//   O = sum_s w_s O_s / sum_s w_s,   lse = (M + log2(sum_s w_s)) * ln 2.
// A split that selected nothing has l_s = 0 and weight 0; a token with no row
// at all gets O = 0 and lse = -inf, as in the attention kernel.  The L2 lines
// of a consumed partial row are dropped without being written back.
__global__ void __launch_bounds__(SfaCfg::COMBINE_THREADS)
    sfa_combine_kernel(const __grid_constant__ SfaParams p, int np) {
    using Cfg = SfaCfg;
    // the partials are written by the attention launch this one depends on
    griddep_wait();
    const int t = (int)blockIdx.x;
    const int head = (int)blockIdx.y * (Cfg::COMBINE_THREADS / 32) + (int)(threadIdx.x >> 5);
    const int lane = (int)(threadIdx.x & 31);
    const int nb = (p.K + Cfg::ROWS - 1) / Cfg::ROWS;
    const int64_t total = (int64_t)p.T * nb;
    const int pf = pair_of_block(total, (int64_t)t * nb, np);
    const int pl = pair_of_block(total, (int64_t)(t + 1) * nb - 1, np);
    if (pf == pl || head >= p.H) return;     // a whole token is finished by its pair
    const int S = pl - pf + 1;
    const int crank = head >> 6, hl = head & 63;
    // slot of split si: its pair's first segment (side 0) unless that pair started in
    // an earlier token (then token t is its last segment, side 1)
    auto slot = [&](int si) -> const uint8_t* {
        const int side = (si == 0 && pair_start(total, pf, np) < (int64_t)t * nb) ? 1 : 0;
        return p.part + ((int64_t)(2 * (pf + si) + side) * 2 + crank) * Cfg::SLOT_BYTES;
    };
    float2 ml = make_float2(-INFINITY, 0.0f);
    if (lane < S) ml = __ldcg(reinterpret_cast<const float2*>(slot(lane) + Cfg::SLOT_O) + hl);
    float M = ml.x;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, d));
    const float w = (M == -INFINITY || ml.x == -INFINITY || !(ml.y > 0.0f)) ? 0.0f : exp2f(ml.x - M) * ml.y;
    float Lsum = w;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, d);
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
#pragma unroll 4
    for (int si = 0; si < S; ++si) {
        const float ws = __shfl_sync(0xffffffffu, w, si);
        const uint4* row = reinterpret_cast<const uint4*>(slot(si) + (int64_t)hl * 1024) + 2 * lane;
        const uint4 x0 = __ldcs(row), x1 = __ldcs(row + 1);
        const uint32_t xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            acc[2 * e] = fmaf(ws, __uint_as_float(xs[e] << 16), acc[2 * e]);
            acc[2 * e + 1] = fmaf(ws, __uint_as_float(xs[e] & 0xFFFF0000u), acc[2 * e + 1]);
        }
    }
    const float inv = Lsum > 0.0f ? 1.0f / Lsum : 0.0f;
    uint4* dst = reinterpret_cast<uint4*>(p.out + ((int64_t)t * p.H + head) * kDv) + 2 * lane;
    dst[0] = make_uint4(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv),
                        pack_bf16(acc[4] * inv, acc[5] * inv), pack_bf16(acc[6] * inv, acc[7] * inv));
    dst[1] = make_uint4(pack_bf16(acc[8] * inv, acc[9] * inv), pack_bf16(acc[10] * inv, acc[11] * inv),
                        pack_bf16(acc[12] * inv, acc[13] * inv), pack_bf16(acc[14] * inv, acc[15] * inv));
    if (lane == 0 && p.lse)
        p.lse[(int64_t)t * p.H + head] = Lsum > 0.0f ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
    // every lane's loads have returned (their values are in the output): drop the rows
    __syncwarp();
    for (int li = lane; li < S * 8; li += 32) discard_l2_line(slot(li >> 3) + (int64_t)hl * 1024 + (li & 7) * 128);
}

}  // namespace dsa
