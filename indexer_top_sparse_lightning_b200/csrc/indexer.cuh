// indexer.cuh -- fused Lightning Indexer + Top-K kernel for sm_100a.
//
// One kernel performs the whole index stage the pages describe as a single
// fused operator ("Large Model Inference Acceleration: Day-0 Adaptation and
// Performance Optimization for New Architectures", section 1.1 "Indexer
// Fusion: Three Kernels into One"; "Day0 Adaptation and Sparse Attention
// Optimization for Long-Sequence LLM Inference", section 4): it reads the
// paged indexer-key cache in place, scores every visible position, applies
// the head weights, selects the Top-K and writes only the index list.
//
//   score(t, s) = sum_h w[t,h] * max(0, q[t,h,:] . k[s,:])
//
// Roles inside a CTA (warp specialised, mbarrier pipelines):
//   warps 0-3  epilogue: TMEM -> registers, ReLU, head-weighted sum in fp32,
//              scores into shared memory, then the radix Top-K select
//   warp 4     TMA producer: walks the block table, loads 128-key tiles
//              (two 64-token pages) with cp.async.bulk.tensor into a
//              128-byte-swizzled ring of shared-memory stages
//   warp 5     TMEM allocator and tcgen05.mma issuer:
//              D[key, (token,head)] = K_tile[128 x D_I] . Q^T, fp32 in TMEM,
//              double-buffered so the epilogue of tile i overlaps the MMA of
//              tile i+1
//   warps 6-9  (fp8 keys only) widen e4m3 codes to bf16 in shared memory;
//              the per-64-element scales are applied in the fp32 epilogue
//
// Top-K: scores never leave shared memory.  A CTA, or a group of CTAs that
// share one sequence, finds the exact K-th largest order-preserving key with
// three radix passes (11/11/10 bits); the CTAs of a group add their
// histograms into a small global histogram and meet at a bounded group
// barrier.  Elements above the threshold are taken; elements equal to it are
// taken lowest position first.  Indices are emitted in ascending position
// order with warp ballots and prefix counts (no atomics on the output).
#pragma once
#include "common.h"
#include "ptx.cuh"
#include "select.cuh"

namespace dsa {

__host__ __device__ constexpr int pow2_at_least(int v) {
    int p = 32;
    while (p < v) p <<= 1;
    return p;
}

// FP8: e4m3 key codes, widened to bf16 in shared memory.  MX (with FP8): MXFP8
// queries and keys -- each code times the power-of-two scale of its 32-element
// group, applied exactly while widening (queries: while building the Q tile), so
// the contraction and one accumulator are those of bf16 keys.
template <bool FP8, int HI, int DI, int NQ, bool MX = false>
struct IdxCfg {
    static_assert(!MX || FP8, "MXFP8 keys are e4m3 codes");
    static constexpr int KB = DI / 64;                        // 64-wide K blocks
    static constexpr int N = (NQ * HI < 16) ? 16 : NQ * HI;   // MMA N (token-major heads)
    static constexpr int ACC = (FP8 && !MX) ? KB : 1;         // fp8 with fp32 scales: one accumulator per scale group
    static constexpr int COLS_BUF = N * ACC;
    static constexpr int TMEM_COLS = pow2_at_least(2 * COLS_BUF);
    // key stages in flight: fp8 keys keep three (their widened copies take two more
    // buffers), so that a CTA holds 16 K scores and a 128 K-context batch of eight
    // plans into one grouped launch
    static constexpr int NSTAGE = FP8 ? 3 : (NQ == 1 ? 4 : 3);
    static constexpr int CODE_BYTES = kTileKeys * DI * (FP8 ? 1 : 2);   // one tile of keys
    // MXFP8: the tile's scale bytes follow its codes in the stage ([128 keys][D_I/32])
    static constexpr int KSC_BYTES = MX ? kTileKeys * (DI / 32) : 0;
    static constexpr int STAGE_BYTES = ((CODE_BYTES + KSC_BYTES + 1023) / 1024) * 1024;
    static constexpr int NCONV = FP8 ? 2 : 0;                 // widened-operand buffers
    static constexpr int NCV = FP8 ? 2 : 1;                   // (modulus for the ring index)
    static constexpr int CONV_BYTES = kTileKeys * DI * 2;
    static constexpr int Q_BYTES = N * DI * 2;
    static constexpr int Q_TX = NQ * HI * DI * 2;             // bytes one Q load brings in
    static constexpr bool Q_PAD = NQ * HI < N;                // rows [NQ*HI, N) stay zero
    static constexpr int HIST_WORDS = kBins;                  // select histograms
    static constexpr int W_FLOATS = NQ * HI;
    // warps 0-7 epilogue and Top-K, 8 TMA producer, 9 MMA issuer, 10-15 fp8 widening
    static constexpr int THREADS = kEpiThreads + 64 + (FP8 ? kConvThreads : 0);
    static constexpr int PRODUCER_WARP = kEpiWarps;
    static constexpr int MMA_WARP = kEpiWarps + 1;
    static constexpr int CONV_WARP0 = kEpiWarps + 2;
    // heads split between the two warps of a TMEM lane quarter (HI >= 32), else one warp
    static constexpr bool SPLIT = HI >= 32;
    static constexpr int HH = SPLIT ? HI / 2 : HI;            // heads per epilogue thread
    static constexpr uint32_t IDESC = idesc_bf16_f32(128, N, false, false);

    static constexpr int OFF_STAGE = 0;
    static constexpr int OFF_CONV = OFF_STAGE + NSTAGE * STAGE_BYTES;
    static constexpr int OFF_Q = OFF_CONV + NCONV * CONV_BYTES;
    static constexpr int OFF_HIST = OFF_Q + Q_BYTES;
    static constexpr int OFF_W = OFF_HIST + HIST_WORDS * 4;
    static constexpr int OFF_MISC = OFF_W + ((W_FLOATS * 4 + 127) / 128) * 128;
    static constexpr int MISC_BYTES = 1024;
    static constexpr int MAX_PAGES = 512;                     // page ids of one work item, staged in smem
    static constexpr int OFF_BLK = OFF_MISC + MISC_BYTES;
    // partial head sums handed between the two warps of a lane quarter, [2][NQ][128]
    static constexpr int OFF_PART = OFF_BLK + MAX_PAGES * 4;
    static constexpr int OFF_LIST = OFF_PART + (SPLIT ? 2 * NQ * kTileKeys * 4 : 0);   // select list, u32 [kListCap]
    static constexpr int OFF_SCORE = OFF_LIST + kListCap * 4;
    // shared memory free during grouped select (the key stages and widened keys)
    static constexpr int SCRATCH_BYTES = OFF_Q - OFF_STAGE;
    // dynamic shared memory = 1024 (alignment slack) + OFF_SCORE + score_cap * 4
    static constexpr int FIXED_SMEM = 1024 + OFF_SCORE;
};

struct IdxMisc {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t conv_full[2];
    uint64_t conv_empty[2];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t q_full;
    uint64_t q_empty;
    uint64_t drain;
    uint64_t gbar;            // grouped select: all published keys of a token landed
    uint32_t tmem_base;
    int abort;
    uint32_t inject;          // test hook: fault injection bits (workspace status area, word 2)
    uint64_t wait_ns;         // bounded-wait limit of this launch
    // mode-0 assignment of this CTA
    int g_valid, g_b, g_rank, g_size, g_tile_begin, g_tile_count, g_group, g_t0, g_nq;
    int64_t g_L;
    SelectSmem sel;
};

// One unit of work: a group of query tokens of one sequence and a chunk of
// its key tiles.
struct IdxItem {
    int b, t0, nq, rank, G, group;
    int tile_begin, tile_count;
    int64_t L;
    int64_t pos[4];
};

template <int NQ>
__device__ __forceinline__ bool get_item(const IndexerParams& p, const IdxMisc* m, int k, IdxItem& it) {
    if (p.mode == 0) {
        if (k != 0 || !m->g_valid) return false;
        it.b = m->g_b;
        it.rank = m->g_rank;
        it.G = m->g_size;
        it.group = m->g_group;
        it.tile_begin = m->g_tile_begin;
        it.tile_count = m->g_tile_count;
        it.t0 = m->g_t0;
        it.nq = m->g_nq;
        it.L = m->g_L;      // keys visible to the window's last token
        for (int j = 0; j < NQ; ++j) it.pos[j] = it.L - it.nq + j;
        return true;
    }
    // mode 1: zig-zag over tokens -- even rounds ascend, odd rounds descend
    const int C = gridDim.x;
    const int local = (k & 1) ? (k * C + (C - 1 - (int)blockIdx.x)) : (k * C + (int)blockIdx.x);
    const int t = p.t_begin + local;
    if (local < 0 || t >= p.t_end) return false;
    // sequence of token t
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(p.cu_q + mid) <= t) lo = mid; else hi = mid - 1;
    }
    it.b = lo;
    it.t0 = t;
    it.nq = 1;
    it.rank = 0;
    it.G = 1;
    it.group = 0;
    it.L = __ldg(p.seq_lens + lo);
    const int nqb = __ldg(p.cu_q + lo + 1) - __ldg(p.cu_q + lo);
    it.pos[0] = it.L - nqb + (t - __ldg(p.cu_q + lo));
    if (it.L > (int64_t)p.max_blocks * kPage || it.pos[0] < 0 || it.pos[0] >= p.score_cap) {
        // inconsistent lengths: report and give this token an empty key range
        set_status(p.status, kStBounds);
        it.L = 0;
        it.pos[0] = -1;
    }
    for (int j = 1; j < NQ; ++j) it.pos[j] = -1;
    it.tile_begin = 0;
    it.tile_count = (int)((it.pos[0] + kTileKeys) / kTileKeys);
    return true;
}

// Calls f(b, t0, n, L) for the query windows [w_begin, w_end) of a mode-0 launch, in
// order: sequence b, its tokens t0 .. t0+n-1, and L = the number of positions the
// window's last token sees.  Window w of sequence b holds its tokens w*nq_max ..; a
// sequence without tokens counts as one window with n = 0 (reported by the caller).
template <typename F>
static __device__ void for_windows(const IndexerParams& p, int nq_max, F&& f) {
    if (p.seq_windows) {
        for (int b = p.w_begin; b < p.w_end; ++b) {
            const int t0 = __ldg(p.cu_q + b);
            f(b, t0, __ldg(p.cu_q + b + 1) - t0, (int64_t)__ldg(p.seq_lens + b));
        }
        return;
    }
    int gi = 0;
    for (int b = 0; b < p.B && gi < p.w_end; ++b) {
        const int t0 = __ldg(p.cu_q + b), nq = __ldg(p.cu_q + b + 1) - t0;
        const int nw = nq >= 1 ? (nq + nq_max - 1) / nq_max : 1;
        if (gi + nw <= p.w_begin) {
            gi += nw;
            continue;
        }
        const int64_t L = __ldg(p.seq_lens + b);
        for (int w = 0; w < nw && gi < p.w_end; ++w, ++gi) {
            if (gi < p.w_begin) continue;
            const int j0 = w * nq_max;
            const int n = nq >= 1 ? (nq - j0 < nq_max ? nq - j0 : nq_max) : 0;
            f(b, t0 + j0, n, L - nq + j0 + n);
        }
    }
}

// Mode-0 partition: every CTA computes the same split of CTAs over the windows
// of the launch, proportional to their key tiles.
static __device__ void assign_groups(const IndexerParams& p, IdxMisc* m, int nq_max, int score_cap) {
    const int C = gridDim.x;
    int64_t total = 0;
    int Wn = 0;
    for_windows(p, nq_max, [&](int, int, int, int64_t L) {
        total += (L + kTileKeys - 1) / kTileKeys;
        ++Wn;
    });
    m->g_valid = 0;
    if (total <= 0 || C < Wn) return;
    int acc = 0, gidx = 0;
    bool done = false;
    for_windows(p, nq_max, [&](int b, int t0, int nq, int64_t L) {
        if (done) return;
        const int tiles = (int)((L + kTileKeys - 1) / kTileKeys);
        int g = 1 + (int)(((int64_t)(C - Wn) * tiles) / total);
        if (g > tiles) g = tiles;
        if (g < 1) g = 1;
        if ((int)blockIdx.x >= acc && (int)blockIdx.x < acc + g) {
            done = true;
            const int r = (int)blockIdx.x - acc;
            const int base = tiles / g, rem = tiles % g;
            const int max_chunk = (base + (rem ? 1 : 0)) * kTileKeys;
            if (nq < 1 || nq > nq_max || nq > L || t0 < 0 || t0 + nq > p.T || L > (int64_t)p.max_blocks * kPage) {
                set_status(p.status, kStBounds);
                return;
            }
            if ((int64_t)max_chunk * nq > score_cap) {
                set_status(p.status, kStCapacity);
                return;
            }
            m->g_valid = 1;
            m->g_b = b;
            m->g_t0 = t0;
            m->g_nq = nq;
            m->g_L = L;
            m->g_rank = r;
            m->g_size = g;
            m->g_group = gidx;
            m->g_tile_begin = r * base + (r < rem ? r : rem);
            m->g_tile_count = base + (r < rem ? 1 : 0);
        }
        acc += g;
        ++gidx;
    });
}

template <bool FP8, int HI, int DI, int NQ, bool MX = false>
__global__ void __launch_bounds__(IdxCfg<FP8, HI, DI, NQ, MX>::THREADS, 1)
    indexer_topk_kernel(const __grid_constant__ IndexerParams p, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k) {
    using Cfg = IdxCfg<FP8, HI, DI, NQ, MX>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_shared(smem_raw, 1024);
    uint8_t* s_stage = smem + Cfg::OFF_STAGE;
    uint8_t* s_conv = smem + Cfg::OFF_CONV;
    uint8_t* s_q = smem + Cfg::OFF_Q;
    uint32_t* s_hist = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_HIST);
    float* s_w = reinterpret_cast<float*>(smem + Cfg::OFF_W);
    IdxMisc* m = reinterpret_cast<IdxMisc*>(smem + Cfg::OFF_MISC);
    float* s_score = reinterpret_cast<float*>(smem + Cfg::OFF_SCORE);
    uint32_t* s_list = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_LIST);
    volatile int* abort = &m->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < Cfg::NSTAGE; ++i) {
            mbar_init(&m->full[i], 1);
            mbar_init(&m->empty[i], FP8 ? kConvThreads : 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&m->conv_full[i], kConvThreads);
            mbar_init(&m->conv_empty[i], 1);
            mbar_init(&m->tfull[i], 1);
            mbar_init(&m->tempty[i], kEpiThreads);
        }
        mbar_init(&m->q_full, MX ? kEpiThreads : 1);   // MXFP8: the epilogue threads build Q
        mbar_init(&m->q_empty, 1);
        mbar_init(&m->drain, 1);
        mbar_init(&m->gbar, 1);
        m->sel.gphase = 0;
        m->abort = 0;
        // test hooks in the status area: word 1 = wait limit in microseconds
        // (0: the default), word 2 = fault injection bits
        const uint32_t us = __ldcg(p.status + 1);
        m->wait_ns = us ? (uint64_t)us * 1000u : kWaitTimeoutNs;
        m->inject = __ldcg(p.status + 2);
        fence_mbar_init();
        if (p.mode == 0) assign_groups(p, m, NQ, p.score_cap);
    }
    if (warp == Cfg::MMA_WARP) {
        tmem_alloc(&m->tmem_base, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == Cfg::PRODUCER_WARP && lane == 0) {
        if (!MX) prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
    }
    if (Cfg::Q_PAD) {
        // MMA rows beyond the real heads read zeros (the Q loads never touch them)
        for (int i = threadIdx.x; i < Cfg::Q_BYTES / 16; i += blockDim.x)
            reinterpret_cast<uint4*>(s_q)[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = m->tmem_base;
    const uint64_t wlim = m->wait_ns;
    // the attention launch that follows may be scheduled now: its CTAs take the SMs
    // this grid leaves and run their prologue before waiting for the index list
    griddep_launch_dependents();

    if (warp == Cfg::PRODUCER_WARP) {
        // ---------------------------------------------------------------- TMA producer
        int32_t* s_blk = reinterpret_cast<int32_t*>(smem + Cfg::OFF_BLK);
        const uint64_t pol = policy_evict_first();
        uint32_t it = 0;
        IdxItem item;
        for (int k = 0; get_item<NQ>(p, m, k, item); ++k) {
            // the page ids of this chunk, staged with one coalesced warp load
            const int64_t npages = (item.L + kPage - 1) / kPage;
            const int pg0 = item.tile_begin * 2;
            int npg = item.tile_count * 2;
            if (pg0 + npg > npages) npg = (int)(npages - pg0);
            if (npg > Cfg::MAX_PAGES) {
                set_status(p.status, kStCapacity);
                npg = Cfg::MAX_PAGES;
            }
            __syncwarp();
            for (int i = lane; i < npg; i += 32) {
                int bid = __ldg(p.block_table + (int64_t)item.b * p.max_blocks + pg0 + i);
                if (bid < 0 || bid >= p.num_blocks) {
                    set_status(p.status, kStBounds);
                    bid = -1;   // out-of-range coordinate: TMA fills zeros
                }
                s_blk[i] = bid;
            }
            __syncwarp();
            int ok = 1;
            if (lane == 0) {
                if (!MX) {
                    if (!mbar_wait(&m->q_empty, (k & 1) ^ 1, abort, wlim)) ok = 0;
                    if (ok) {
                        mbar_arrive_expect_tx(&m->q_full, Cfg::Q_TX);
                        for (int kb = 0; kb < Cfg::KB; ++kb)
                            tma_load_3d(s_q + kb * Cfg::N * 128, &tm_q, &m->q_full, kb * 64, 0, item.t0);
                    }
                }
                for (int li = 0; ok && li < item.tile_count; ++li, ++it) {
                    const int s = it % Cfg::NSTAGE;
                    if (!mbar_wait(&m->empty[s], ((it / Cfg::NSTAGE) & 1) ^ 1, abort, wlim)) { ok = 0; break; }
                    int blk[2];
                    int nvalid = 0;
                    for (int pp = 0; pp < 2; ++pp) {
                        const int i = li * 2 + pp;
                        blk[pp] = i < npg ? s_blk[i] : -2;
                        nvalid += i < npg;
                    }
                    uint8_t* st = s_stage + s * Cfg::STAGE_BYTES;
                    // MXFP8: a page's 64 scale words come along by one bulk copy (none for an
                    // out-of-range page, whose codes read as zeros)
                    constexpr uint32_t PSC = kPage * (DI / 32);
                    uint32_t sc_bytes = 0;
                    if (MX)
                        for (int pp = 0; pp < 2; ++pp) sc_bytes += blk[pp] >= 0 ? PSC : 0u;
                    mbar_arrive_expect_tx(&m->full[s], nvalid * kPage * DI * (FP8 ? 1 : 2) + sc_bytes);
                    for (int pp = 0; pp < 2; ++pp) {
                        if (blk[pp] == -2) continue;
                        if (FP8) {
                            tma_load_2d_hint(st + pp * kPage * DI, &tm_k, &m->full[s], 0, blk[pp] * kPage, pol);
                            if (MX && blk[pp] >= 0)
                                bulk_load(st + Cfg::CODE_BYTES + pp * PSC, p.k_scale_e8 + (int64_t)blk[pp] * PSC, PSC,
                                          &m->full[s]);
                        } else {
                            for (int kb = 0; kb < Cfg::KB; ++kb)
                                tma_load_2d_hint(st + kb * (kTileKeys * 128) + pp * (kPage * 128), &tm_k,
                                                 &m->full[s], kb * 64, blk[pp] * kPage, pol);
                        }
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
        }
        // drain: no TMA write may still be in flight when the CTA exits
        if (lane == 0) {
            const uint32_t first = it > (uint32_t)Cfg::NSTAGE ? it - Cfg::NSTAGE : 0u;
            volatile int no_abort = 0;
            for (uint32_t d = first; d < it; ++d)
                mbar_wait(&m->full[d % Cfg::NSTAGE], (d / Cfg::NSTAGE) & 1, &no_abort, wlim);
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t it = 0;
            IdxItem item;
            bool ok = true;
            for (int k = 0; ok && get_item<NQ>(p, m, k, item); ++k) {
                if (!mbar_wait(&m->q_full, k & 1, abort, wlim)) break;
                tc_fence_after();
                for (int li = 0; li < item.tile_count; ++li, ++it) {
                    const int buf = it & 1;
                    const uint8_t* a_base;
                    if (FP8) {
                        const int cb = it % Cfg::NCV;
                        if (!mbar_wait(&m->conv_full[cb], (it / Cfg::NCV) & 1, abort, wlim)) { ok = false; break; }
                        a_base = s_conv + cb * Cfg::CONV_BYTES;
                    } else {
                        const int s = it % Cfg::NSTAGE;
                        if (!mbar_wait(&m->full[s], (it / Cfg::NSTAGE) & 1, abort, wlim)) { ok = false; break; }
                        a_base = s_stage + s * Cfg::STAGE_BYTES;
                    }
                    if (!mbar_wait(&m->tempty[buf], ((it >> 1) & 1) ^ 1, abort, wlim)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(a_base);
                    const uint32_t b_addr = smem_u32(s_q);
#pragma unroll
                    for (int kb = 0; kb < Cfg::KB; ++kb) {
#pragma unroll
                        for (int k16 = 0; k16 < 4; ++k16) {
                            const uint64_t ad = sdesc_sw128(a_addr + kb * (kTileKeys * 128) + k16 * 32, 16, 1024);
                            const uint64_t bd = sdesc_sw128(b_addr + kb * (Cfg::N * 128) + k16 * 32, 16, 1024);
                            const uint32_t d = tmem_base + buf * Cfg::COLS_BUF + (Cfg::ACC > 1 ? kb * Cfg::N : 0);
                            const uint32_t acc = Cfg::ACC > 1 ? (k16 > 0) : (kb > 0 || k16 > 0);
                            umma_bf16(d, ad, bd, Cfg::IDESC, acc);
                        }
                    }
                    if (FP8) umma_commit(&m->conv_empty[it % Cfg::NCV]);
                    else umma_commit(&m->empty[it % Cfg::NSTAGE]);
                    umma_commit(&m->tfull[buf]);
                }
                umma_commit(&m->q_empty);
            }
            // drain: every issued MMA completes before TMEM is released
            umma_commit(&m->drain);
            volatile int no_abort = 0;
            mbar_wait(&m->drain, 0, &no_abort, wlim);
        }
    } else if (FP8 && warp >= Cfg::CONV_WARP0) {
        // ---------------------------------------------------------------- fp8 -> bf16 widening
        // MXFP8 keys: each 16-code chunk lies in one 32-element group, whose power-of-two
        // scale multiplies the codes exactly before the (exact) conversion to bf16.
        const int ct = threadIdx.x - Cfg::CONV_WARP0 * 32;
        uint32_t it = 0;
        IdxItem item;
        bool ok = true;
        constexpr int CH = DI / 16;   // 16-byte chunks of codes per key
        for (int k = 0; ok && get_item<NQ>(p, m, k, item); ++k) {
            for (int li = 0; li < item.tile_count; ++li, ++it) {
                const int s = it % Cfg::NSTAGE;
                const int cb = it % Cfg::NCV;
                if (!mbar_wait(&m->full[s], (it / Cfg::NSTAGE) & 1, abort, wlim)) { ok = false; break; }
                if (!mbar_wait(&m->conv_empty[cb], ((it / Cfg::NCV) & 1) ^ 1, abort, wlim)) { ok = false; break; }
                const uint8_t* raw = s_stage + s * Cfg::STAGE_BYTES;
                uint8_t* dst = s_conv + cb * Cfg::CONV_BYTES;
#pragma unroll 4
                for (int u = ct; u < kTileKeys * CH; u += kConvThreads) {
                    const int r = u / CH, c = u % CH;
                    const uint4 v = *reinterpret_cast<const uint4*>(raw + r * DI + c * 16);
                    float sc = 1.0f;
                    if (MX) {
                        // scale byte of group c/2 of key r (rows of a page past the sequence
                        // hold whatever the stage held; their keys are never selected)
                        const uint32_t e = raw[Cfg::CODE_BYTES + r * (DI / 32) + (c >> 1)];
                        sc = e ? __uint_as_float(e << 23) : __uint_as_float(0x00400000u);   // 2^(e - 127)
                    }
                    uint32_t outw[8];
                    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        uint32_t h01, h23;
                        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h01) : "h"((uint16_t)(in[e] & 0xFFFFu)));
                        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h23) : "h"((uint16_t)(in[e] >> 16)));
                        float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
                        float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
                        if (MX) {
                            f01.x *= sc;
                            f01.y *= sc;
                            f23.x *= sc;
                            f23.y *= sc;
                        }
                        const __nv_bfloat162 b01 = __float22bfloat162_rn(f01);
                        const __nv_bfloat162 b23 = __float22bfloat162_rn(f23);
                        outw[2 * e] = *reinterpret_cast<const uint32_t*>(&b01);
                        outw[2 * e + 1] = *reinterpret_cast<const uint32_t*>(&b23);
                    }
                    const int kb = c >> 2;
                    const int q0 = (c & 3) * 2;
                    uint8_t* row = dst + kb * (kTileKeys * 128) + r * 128;
                    *reinterpret_cast<uint4*>(row + ((q0 ^ (r & 7)) << 4)) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
                    *reinterpret_cast<uint4*>(row + (((q0 + 1) ^ (r & 7)) << 4)) =
                        make_uint4(outw[4], outw[5], outw[6], outw[7]);
                }
                fence_proxy_async_smem();
                mbar_arrive(&m->conv_full[cb]);
                mbar_arrive(&m->empty[s]);
            }
        }
    } else if (warp < kEpiWarps) {
        // ---------------------------------------------------------------- epilogue + select
        // Warps w and w+4 read the same TMEM lanes (key rows 32*(w%4)..): with SPLIT each
        // sums half of the heads and warp w adds warp w+4's partial; otherwise warps 4-7
        // wait out the epilogue.  All eight warps run the Top-K.
        const int row = 32 * (warp & 3) + lane;   // TMEM lane == key row in the tile
        const int half = warp >> 2;
        const bool scorer = Cfg::SPLIT || half == 0;
        const bool owner = half == 0;              // writes the final score of its row
        float* s_part = reinterpret_cast<float*>(smem + Cfg::OFF_PART);
        uint32_t it = 0;
        IdxItem item;
        bool ok = true;
        for (int k = 0; ok && get_item<NQ>(p, m, k, item); ++k) {
            for (int i = threadIdx.x; i < NQ * HI; i += kEpiThreads) {
                const int j = i / HI;
                s_w[i] = (j < item.nq) ? __ldg(p.w + (int64_t)(item.t0 + j) * HI + (i % HI)) : 0.0f;
            }
            if (threadIdx.x < NQ) {
                m->sel.kmin[threadIdx.x] = 0xFFFFFFFFu;
                m->sel.kmax[threadIdx.x] = 0u;
            }
            if (MX) {
                // MXFP8 queries: once the previous item's MMAs are done with Q, build the
                // bf16 Q tile (128-byte swizzled, token-major heads) from the codes, each
                // times the power-of-two scale of its 32-element group (exact)
                if (mbar_wait(&m->q_empty, (k & 1) ^ 1, abort, wlim)) {
                    constexpr int CPR = DI / 8;   // 16-byte bf16 units per head row
                    for (int u = threadIdx.x; u < NQ * HI * CPR; u += kEpiThreads) {
                        const int r = u / CPR, c = u % CPR;
                        const int j = r / HI, h = r % HI;
                        uint32_t outw[4] = {0u, 0u, 0u, 0u};
                        if (j < item.nq) {
                            const int64_t qi = (int64_t)(item.t0 + j) * HI + h;
                            const uint2 v = __ldg(reinterpret_cast<const uint2*>(p.q_codes + qi * DI + c * 8));
                            const uint32_t e = __ldg(p.q_scale + qi * (DI / 32) + (c * 8) / 32);
                            const float sc = e ? __uint_as_float(e << 23) : __uint_as_float(0x00400000u);
                            const uint32_t in[2] = {v.x, v.y};
#pragma unroll
                            for (int e2 = 0; e2 < 2; ++e2) {
                                uint32_t h01, h23;
                                asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h01) : "h"((uint16_t)(in[e2] & 0xFFFFu)));
                                asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h23) : "h"((uint16_t)(in[e2] >> 16)));
                                float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
                                float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
                                f01.x *= sc;
                                f01.y *= sc;
                                f23.x *= sc;
                                f23.y *= sc;
                                const __nv_bfloat162 b01 = __float22bfloat162_rn(f01);
                                const __nv_bfloat162 b23 = __float22bfloat162_rn(f23);
                                outw[2 * e2] = *reinterpret_cast<const uint32_t*>(&b01);
                                outw[2 * e2 + 1] = *reinterpret_cast<const uint32_t*>(&b23);
                            }
                        }
                        // 64-element K block c/8, 16-byte unit c%8 of the row, swizzled by row
                        *reinterpret_cast<uint4*>(s_q + (c >> 3) * (Cfg::N * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4)) =
                            make_uint4(outw[0], outw[1], outw[2], outw[3]);
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&m->q_full);
            }
            GroupView gv{nullptr, nullptr, nullptr, item.G, item.rank};
            uint32_t gen = 0;
            if (item.G > 1) {
                uint8_t* gw = p.group_ws + (int64_t)item.group * p.group_ws_stride;
                gv.sync = reinterpret_cast<uint32_t*>(gw);
                gv.hdr = reinterpret_cast<uint32_t*>(gw + 128);
                // published-key slots of this group's CTAs (contiguous, rank order)
                gv.cand = p.cand + (int64_t)((int)blockIdx.x - item.rank) * p.cand_slot;
                // the group's barrier generation cannot move before this CTA arrives
                if (threadIdx.x == 0) gen = ld_acquire_gpu(gv.sync + 1);
            }
            named_bar_sync(1, kEpiThreads);
            const int stride = item.tile_count * kTileKeys;   // score slots per token
            const int64_t chunk0 = (int64_t)item.tile_begin * kTileKeys;
            uint32_t kmn[NQ], kmx[NQ];
#pragma unroll
            for (int j = 0; j < NQ; ++j) {
                kmn[j] = 0xFFFFFFFFu;
                kmx[j] = 0u;
            }
            const int64_t npages = (item.L + kPage - 1) / kPage;
            for (int li = 0; li < item.tile_count; ++li, ++it) {
                const int buf = it & 1;
                const int64_t pos = chunk0 + (int64_t)li * kTileKeys + row;
                float sc[2] = {1.0f, 1.0f};
                if (FP8 && !MX && scorer) {     // fp32 group scales, applied to the accumulators
                    const int64_t pg = pos / kPage;
                    if (pg < npages) {
                        const int bid = __ldg(p.block_table + (int64_t)item.b * p.max_blocks + pg);
                        if (bid >= 0 && bid < p.num_blocks) {
                            const float* sp = p.k_scale + ((int64_t)bid * kPage + pos % kPage) * Cfg::KB;
                            sc[0] = __ldg(sp);
                            if (Cfg::KB > 1) sc[1] = __ldg(sp + 1);
                        }
                    }
                }
                const bool got = mbar_wait(&m->tfull[buf], (it >> 1) & 1, abort, wlim);
                float score[NQ];
#pragma unroll
                for (int j = 0; j < NQ; ++j) score[j] = 0.0f;
                if (got) {
                    tc_fence_after();
                    const uint32_t tb = tmem_base + ((uint32_t)((warp & 3) * 32) << 16) + buf * Cfg::COLS_BUF;
#pragma unroll
                    for (int j = 0; j < NQ; ++j) {
                        if (!scorer || j >= item.nq) continue;
                        // four independent partial sums (head h into sum h % 4), weights
                        // read four at a time
                        float part[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                        constexpr int CW = Cfg::HH < 32 ? Cfg::HH : 32;
#pragma unroll
                        for (int c0 = 0; c0 < Cfg::HH; c0 += CW) {
                            uint32_t a0[32], a1[32];
                            const int h0 = (Cfg::SPLIT ? half * Cfg::HH : 0) + c0;   // first head of the chunk
                            const uint32_t col = j * HI + h0;
                            if constexpr (CW == 32) {
                                tmem_ld32(tb + col, a0);
                                if (Cfg::ACC > 1) tmem_ld32(tb + Cfg::N + col, a1);
                            } else if constexpr (CW == 16) {
                                tmem_ld16(tb + col, *reinterpret_cast<uint32_t(*)[16]>(a0));
                                if (Cfg::ACC > 1) tmem_ld16(tb + Cfg::N + col, *reinterpret_cast<uint32_t(*)[16]>(a1));
                            } else {
                                tmem_ld8(tb + col, *reinterpret_cast<uint32_t(*)[8]>(a0));
                                if (Cfg::ACC > 1) tmem_ld8(tb + Cfg::N + col, *reinterpret_cast<uint32_t(*)[8]>(a1));
                            }
                            tmem_wait_ld();
                            const float4* w4 = reinterpret_cast<const float4*>(s_w + j * HI + h0);
#pragma unroll
                            for (int h = 0; h < CW; h += 4) {
                                const float4 wv = w4[h >> 2];
                                const float wq[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    float x = __uint_as_float(a0[h + e]);
                                    if (Cfg::ACC > 1) {
                                        x = x * sc[0];
                                        x = fmaf(__uint_as_float(a1[h + e]), sc[1], x);
                                    } else if (FP8 && !MX) {
                                        x = x * sc[0];
                                    }
                                    part[e] = fmaf(wq[e], fmaxf(x, 0.0f), part[e]);
                                }
                            }
                        }
                        score[j] = (part[0] + part[1]) + (part[2] + part[3]);
                    }
                    tc_fence_before();
                    mbar_arrive(&m->tempty[buf]);
                    if (Cfg::SPLIT && !owner) {
#pragma unroll
                        for (int j = 0; j < NQ; ++j) s_part[(buf * NQ + j) * kTileKeys + row] = score[j];
                    }
                }
                // the hand-over barrier carries the exit vote, so every thread leaves together
                const bool all = Cfg::SPLIT ? named_bar_and(2, kEpiThreads, got) : got;
                if (!all) { ok = false; break; }
                if (!owner) continue;
#pragma unroll
                for (int j = 0; j < NQ; ++j) {
                    if (j < item.nq) {
                        float f = score[j];
                        if (Cfg::SPLIT) f += s_part[(buf * NQ + j) * kTileKeys + row];
                        f = f == 0.0f ? 0.0f : f;
                        s_score[j * stride + li * kTileKeys + row] = f;
                        // range of the visible keys, for the select's first histogram
                        if (pos <= item.pos[j]) {
                            const uint32_t key = order_key(f);
                            kmn[j] = min(kmn[j], key);
                            kmx[j] = max(kmx[j], key);
                        }
                    }
                }
            }
            if (!ok) break;
#pragma unroll
            for (int j = 0; j < NQ; ++j) {
#pragma unroll
                for (int o = 16; o; o >>= 1) {
                    kmn[j] = min(kmn[j], __shfl_xor_sync(0xffffffffu, kmn[j], o));
                    kmx[j] = max(kmx[j], __shfl_xor_sync(0xffffffffu, kmx[j], o));
                }
                if (lane == 0 && j < item.nq) {
                    red_min_shared(&m->sel.kmin[j], kmn[j]);
                    red_max_shared(&m->sel.kmax[j], kmx[j]);
                }
            }
            named_bar_sync(1, kEpiThreads);

            // ------------------------------------------------------------ Top-K select
            int nloc[NQ];
            bool active[NQ];
            bool any_active = false;
#pragma unroll
            for (int j = 0; j < NQ; ++j) {
                const int64_t vis = item.pos[j] + 1;      // group-wide visible positions
                int64_t n = vis - chunk0;
                n = n < 0 ? 0 : (n > stride ? stride : n);
                nloc[j] = (j < item.nq) ? (int)n : 0;
                active[j] = (j < item.nq) && vis > p.K;
                any_active |= active[j];
            }
            // take-all tokens: every visible position, in place
#pragma unroll
            for (int j = 0; j < NQ; ++j) {
                if (j >= item.nq || active[j]) continue;
                const int64_t tok = item.t0 + j;
                int32_t* oi = p.out_idx + tok * p.K;
                float* os = p.out_score ? p.out_score + tok * p.K : nullptr;
                for (int i = threadIdx.x; i < nloc[j]; i += kEpiThreads) {
                    oi[chunk0 + i] = (int32_t)(chunk0 + i);
                    if (os) os[chunk0 + i] = s_score[j * stride + i];
                }
                if (item.rank == 0) {
                    for (int64_t i = item.pos[j] + 1 + threadIdx.x; i < p.K; i += kEpiThreads) {
                        oi[i] = -1;
                        if (os) os[i] = -__int_as_float(0x7f800000);
                    }
                }
            }
            if (any_active &&
                !topk_select<NQ>(p, gv, gen, s_score, stride, nloc, active, chunk0, item.t0, s_hist, s_list,
                                 smem + Cfg::OFF_STAGE, Cfg::SCRATCH_BYTES, &m->sel,
                                 abort, wlim, m->inject, &m->gbar)) {
                ok = false;
                break;
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == Cfg::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
    if (threadIdx.x == 0 && m->abort) set_status(p.status, kStTimeout);
}

}  // namespace dsa
