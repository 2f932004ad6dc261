// select.cuh -- exact Top-K of shared-memory score rows, within a CTA or
// across a group of CTAs that share one sequence (sm_100a).
//
// The Top-K pass of the fused indexer ("Large Model Inference Acceleration:
// Day-0 Adaptation and Performance Optimization for New Architectures",
// section 1.1: after scoring, data stays in vector registers or shared
// memory for the weighted aggregation and the Top-K pass; no intermediate
// tensor goes to global memory).
//
// Scores are mapped to order-preserving 32-bit keys (-0 folded into +0).  The
// K-th largest key T is found with three radix digits (11/11/10 bits); the
// CTAs of a group add their digit histograms into a small global histogram
// and meet at a bounded barrier.  Elements above T are selected; elements
// equal to T are selected lowest position first.  The chunk of a CTA is a
// contiguous position range and warp w of the four select warps owns a
// contiguous quarter of it, so "warp order" is "position order" and every
// count needed for the output offsets is a per-warp running count:
//   pass-1 scan: elements whose first digit is above T's  (counted)
//   pass-2 scan: elements matching the first digit whose second is above
//                (counted); elements matching both digits are listed
//   after T:     listed elements above / equal to T       (counted)
// Indices are written in ascending position order with ballots and prefix
// counts (no atomics on the output).
#pragma once
#include "common.h"
#include "ptx.cuh"

namespace dsa {

constexpr int kListCap = 256;   // listed (two-digit match) elements per warp and token

struct SelectSmem {
    uint32_t scan[8];
    uint32_t wcnt[4][4][2];     // [token][warp][gt, eq]
    uint32_t wallow[4][4];      // [token][warp] tied elements the warp may take
    uint32_t sel_bin[4];
    uint32_t sel_kk[4];
    uint32_t sel_take[4];
    uint32_t sel_base[4];
    uint32_t list_n[4][4];      // [token][warp]
};

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t code) {
    atomicCAS(status, 0u, code);
}

// Bounded barrier among the CTAs of one group (called by the 128 select
// threads).  Sense-reversing: the last arriver resets the count and bumps
// the generation.  `gen` is thread 0's copy of the generation, read once per
// work item and advanced here, so a barrier costs one atomic and the wait.
__device__ bool group_barrier(uint32_t* sync, int G, uint32_t& gen, uint32_t* status, volatile int* abort) {
    named_bar_sync(1, kEpiThreads);
    if (threadIdx.x == 0 && !*abort) {
        uint32_t* count = sync;
        uint32_t* genp = sync + 1;
        const uint32_t old = atom_add_acq_rel_gpu(count, 1u);
        if (old == (uint32_t)G - 1u) {
            *reinterpret_cast<volatile uint32_t*>(count) = 0u;
            st_release_gpu(genp, gen + 1u);
        } else {
            const uint64_t t0 = globaltimer();
            while (ld_acquire_gpu(genp) == gen) {
                if (globaltimer() - t0 > kWaitTimeoutNs) {
                    set_status(status, kStTimeout);
                    *abort = 1;
                    break;
                }
            }
        }
        gen += 1u;
    }
    named_bar_sync(1, kEpiThreads);
    return !*abort;
}

// Exclusive prefix over the 128 select threads; *total receives the sum.
__device__ __forceinline__ uint32_t epi_exclusive_scan(uint32_t v, uint32_t* scratch, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    named_bar_sync(1, kEpiThreads);
    uint32_t before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t s = scratch[w];
        if (w < warp) before += s;
        all += s;
    }
    named_bar_sync(1, kEpiThreads);
    *total = all;
    return before + x - v;
}

// Radix step: the bin of the histogram (nb bins, higher bin = larger keys)
// holding the kk-th largest element, and the rank of that element in the bin.
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nb, uint32_t kk, uint32_t* scratch,
                                         uint32_t* out_bin, uint32_t* out_kk) {
    const int per = nb / kEpiThreads;
    const int hi_bin = nb - 1 - (int)threadIdx.x * per;
    uint32_t s = 0;
    for (int i = 0; i < per; ++i) s += hist[hi_bin - i];
    uint32_t total;
    const uint32_t before = epi_exclusive_scan(s, scratch, &total);
    if (before < kk && kk <= before + s) {
        uint32_t c = before;
        for (int i = 0; i < per; ++i) {
            const uint32_t h = hist[hi_bin - i];
            if (c + h >= kk) {
                *out_bin = (uint32_t)(hi_bin - i);
                *out_kk = kk - c;
                break;
            }
            c += h;
        }
    }
    named_bar_sync(1, kEpiThreads);
}

// Add this CTA's digit histogram (nonzero bins) into the group histogram.
__device__ __forceinline__ void push_hist(const uint32_t* local, uint32_t* global, int nb) {
    for (int i = threadIdx.x; i < nb; i += kEpiThreads) {
        const uint32_t v = local[i];
        if (v) atomicAdd(global + i, v);
    }
}

// Replace the local histogram by the group's: every load in flight at once.
__device__ __forceinline__ void pull_hist(uint32_t* local, const uint32_t* global, int nb) {
    constexpr int V = 2048 / (4 * kEpiThreads);   // uint4 per thread for 2048 bins
    uint4 v[V];
#pragma unroll
    for (int u = 0; u < V; ++u) {
        const int i = (u * kEpiThreads + (int)threadIdx.x) * 4;
        v[u] = i < nb ? __ldcg(reinterpret_cast<const uint4*>(global + i)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < V; ++u) {
        const int i = (u * kEpiThreads + (int)threadIdx.x) * 4;
        if (i < nb) *reinterpret_cast<uint4*>(local + i) = v[u];
    }
}

// Loads 4 x 32 consecutive scores of a warp's range (lane-strided), keyed.
struct KeyBatch {
    uint32_t key[4];
    bool in[4];
};
__device__ __forceinline__ KeyBatch load_keys(const float* s, int i0, int end, int lane) {
    KeyBatch kb;
    float f[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * 32 + lane;
        kb.in[u] = i < end;
        f[u] = kb.in[u] ? s[i] : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) kb.key[u] = order_key(f[u]);
    return kb;
}

struct GroupView {
    uint32_t* sync;     // {count, gen}
    uint32_t* hist;     // [3][NQ][2048]
    uint32_t* cnt;      // [ranks][NQ][2]
    int G, rank;
};

// Exact Top-K of NQ tokens' score rows held in shared memory (s_score, token
// j at j*stride, nloc[j] valid entries starting at position chunk0).
// Writes out_idx/out_score rows [t0 + j] in ascending position order.
// Called by the 128 select threads; the pass-0 (top 11 bits) histogram of
// every visible element must already be in s_hist[j*2048 ...].
template <int NQ>
__device__ bool topk_select(const IndexerParams& p, const GroupView& gv, uint32_t& gen, float* s_score,
                            int stride, const int (&nloc)[NQ], const bool (&active)[NQ], int64_t chunk0,
                            int64_t t0, uint32_t* s_hist, uint16_t* s_list, SelectSmem* sm, volatile int* abort) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t prefix[NQ], kk[NQ];
#pragma unroll
    for (int j = 0; j < NQ; ++j) { prefix[j] = 0; kk[j] = (uint32_t)p.K; }
    // per-warp running counts of elements above the (partial) threshold
    uint32_t wgt[NQ];
#pragma unroll
    for (int j = 0; j < NQ; ++j) wgt[j] = 0;

    auto quarter = [&](int j, int& beg, int& end) {
        const int qlen = ((nloc[j] + 4 * 32 - 1) / (4 * 32)) * 32;
        beg = warp * qlen;
        end = min(nloc[j], beg + qlen);
    };

    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        if (pass > 0) {
            for (int i = threadIdx.x; i < NQ * 2048; i += kEpiThreads) s_hist[i] = 0u;
            named_bar_sync(1, kEpiThreads);
#pragma unroll
            for (int j = 0; j < NQ; ++j) {
                if (!active[j]) continue;
                const float* sj = s_score + j * stride;
                uint32_t* hj = s_hist + j * 2048;
                int beg, end;
                quarter(j, beg, end);
                uint32_t gt = 0, n_list = 0;
                uint16_t* wl = s_list + (j * 4 + warp) * kListCap;
                // pass 1: match the first digit; pass 2: match the first two digits
                const int mshift = pass == 1 ? 21 : 10;
                const uint32_t want = prefix[j] >> mshift;
                const uint32_t d1 = prefix[j] >> 21;
                for (int i0 = beg; i0 < end; i0 += 128) {
                    const KeyBatch kb = load_keys(sj, i0, end, lane);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t hi = kb.key[u] >> mshift;
                        // above the threshold at this digit, and not already counted at the previous one
                        const bool above = hi > want && (pass == 1 || (kb.key[u] >> 21) == d1);
                        gt += __popc(__ballot_sync(0xffffffffu, kb.in[u] && above));
                        const bool match = kb.in[u] && hi == want;
                        if (match) atomicAdd(hj + ((kb.key[u] >> shift) & (nb - 1)), 1u);
                        if (pass == 2) {
                            const uint32_t mm = __ballot_sync(0xffffffffu, match);
                            const uint32_t at = n_list + __popc(mm & lt_mask);
                            if (match && at < kListCap) wl[at] = (uint16_t)(i0 + u * 32 + lane);
                            n_list += __popc(mm);
                        }
                    }
                }
                wgt[j] += gt;
                if (pass == 2 && lane == 0) sm->list_n[j][warp] = n_list;
            }
            named_bar_sync(1, kEpiThreads);
        }
        if (gv.G > 1) {
            uint32_t* gh = gv.hist + pass * NQ * 2048;
#pragma unroll
            for (int j = 0; j < NQ; ++j)
                if (active[j]) push_hist(s_hist + j * 2048, gh + j * 2048, nb);
            if (!group_barrier(gv.sync, gv.G, gen, p.status, abort)) return false;
#pragma unroll
            for (int j = 0; j < NQ; ++j)
                if (active[j]) pull_hist(s_hist + j * 2048, gh + j * 2048, nb);
            // the histogram of the previous pass has been read by every CTA
            if (gv.rank == 0 && pass > 0) {
                uint32_t* prev = gv.hist + (pass - 1) * NQ * 2048;
                for (int i = threadIdx.x * 4; i < NQ * 2048; i += kEpiThreads * 4)
                    *reinterpret_cast<uint4*>(prev + i) = make_uint4(0, 0, 0, 0);
            }
            named_bar_sync(1, kEpiThreads);
        }
#pragma unroll
        for (int j = 0; j < NQ; ++j) {
            if (!active[j]) continue;
            find_bin(s_hist + j * 2048, nb, kk[j], sm->scan, &sm->sel_bin[j], &sm->sel_kk[j]);
            prefix[j] |= sm->sel_bin[j] << shift;
            kk[j] = sm->sel_kk[j];
        }
        if (threadIdx.x == 0) DSA_TRACE_MARK(3 + pass);
    }

    // ---- per-warp counts above / equal to the exact threshold T = prefix
    bool overflow = false;
#pragma unroll
    for (int j = 0; j < NQ; ++j)
        if (active[j])
            for (int w = 0; w < 4; ++w) overflow |= sm->list_n[j][w] > (uint32_t)kListCap;
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
        uint32_t gt = 0, eq = 0;
        if (active[j]) {
            const float* sj = s_score + j * stride;
            if (!overflow) {
                const uint16_t* wl = s_list + (j * 4 + warp) * kListCap;
                const uint32_t n = sm->list_n[j][warp];
                for (uint32_t i = lane; i < n; i += 32) {
                    const uint32_t key = order_key(sj[wl[i]]);
                    gt += key > prefix[j];
                    eq += key == prefix[j];
                }
#pragma unroll
                for (int o = 16; o; o >>= 1) {
                    gt += __shfl_xor_sync(0xffffffffu, gt, o);
                    eq += __shfl_xor_sync(0xffffffffu, eq, o);
                }
                gt += wgt[j];
            } else {
                // too many ties near the threshold for the lists: count directly
                int beg, end;
                quarter(j, beg, end);
                for (int i0 = beg; i0 < end; i0 += 128) {
                    const KeyBatch kb = load_keys(sj, i0, end, lane);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        gt += __popc(__ballot_sync(0xffffffffu, kb.in[u] && kb.key[u] > prefix[j]));
                        eq += __popc(__ballot_sync(0xffffffffu, kb.in[u] && kb.key[u] == prefix[j]));
                    }
                }
            }
            if (lane == 0) {
                sm->wcnt[j][warp][0] = gt;
                sm->wcnt[j][warp][1] = eq;
            }
        }
    }
    named_bar_sync(1, kEpiThreads);
    uint32_t cgt[NQ], ceq[NQ], gt_before[NQ], eq_before[NQ], weq[NQ];
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
        cgt[j] = ceq[j] = gt_before[j] = eq_before[j] = weq[j] = 0;
        if (!active[j]) continue;
        for (int w = 0; w < 4; ++w) {
            const uint32_t g = sm->wcnt[j][w][0], e = sm->wcnt[j][w][1];
            if (w < warp) { gt_before[j] += g; eq_before[j] += e; }
            if (w == warp) weq[j] = e;
            cgt[j] += g;
            ceq[j] += e;
        }
    }
    uint32_t take[NQ], base[NQ];
#pragma unroll
    for (int j = 0; j < NQ; ++j) { take[j] = min(kk[j], ceq[j]); base[j] = 0; }
    if (gv.G > 1) {
        // split the tied elements (lowest positions first, i.e. lower ranks
        // first) and the output offsets across the group
        if (threadIdx.x == 0) {
#pragma unroll
            for (int j = 0; j < NQ; ++j) {
                if (!active[j]) continue;
                __stcg(gv.cnt + (gv.rank * NQ + j) * 2, cgt[j]);
                __stcg(gv.cnt + (gv.rank * NQ + j) * 2 + 1, ceq[j]);
            }
        }
        if (!group_barrier(gv.sync, gv.G, gen, p.status, abort)) return false;
        // counts of the lower ranks: loaded by many threads at once into shared
        // memory (the histogram area is free now), then combined in rank order
        // by one thread, because the tie split depends on the running total
        uint2* cnt_s = reinterpret_cast<uint2*>(s_hist);
        for (int i = threadIdx.x; i < gv.rank * NQ; i += kEpiThreads)
            cnt_s[i] = __ldcg(reinterpret_cast<const uint2*>(gv.cnt) + i);
        named_bar_sync(1, kEpiThreads);
        if (threadIdx.x == 0) {
#pragma unroll
            for (int j = 0; j < NQ; ++j) {
                if (!active[j]) continue;
                uint32_t eqb = 0, ob = 0;
                for (int r = 0; r < gv.rank; ++r) {
                    const uint2 c = cnt_s[r * NQ + j];
                    ob += c.x + (kk[j] > eqb ? min(kk[j] - eqb, c.y) : 0u);
                    eqb += c.y;
                }
                sm->sel_take[j] = kk[j] > eqb ? min(kk[j] - eqb, ceq[j]) : 0u;
                sm->sel_base[j] = ob;
            }
        }
        if (gv.rank == 0) {
            // every CTA of the group has read the last pass's histogram
            uint32_t* last = gv.hist + 2 * NQ * 2048;
            for (int i = threadIdx.x * 4; i < NQ * 2048; i += kEpiThreads * 4)
                *reinterpret_cast<uint4*>(last + i) = make_uint4(0, 0, 0, 0);
        }
        named_bar_sync(1, kEpiThreads);
#pragma unroll
        for (int j = 0; j < NQ; ++j) {
            take[j] = sm->sel_take[j];
            base[j] = sm->sel_base[j];
        }
    }
    if (threadIdx.x == 0) DSA_TRACE_MARK(6);
    // ---- this warp's share of the tied elements, output offsets
    uint32_t allow[NQ];
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
        allow[j] = take[j] > eq_before[j] ? min(take[j] - eq_before[j], weq[j]) : 0u;
        if (lane == 0) sm->wallow[j][warp] = allow[j];
    }
    named_bar_sync(1, kEpiThreads);
    // ---- emission in ascending position order
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
        if (!active[j]) continue;
        uint32_t out = base[j] + gt_before[j];
        for (int w = 0; w < warp; ++w) out += sm->wallow[j][w];
        int beg, end;
        quarter(j, beg, end);
        const float* sj = s_score + j * stride;
        int32_t* oi = p.out_idx + (t0 + j) * p.K;
        float* os = p.out_score ? p.out_score + (t0 + j) * p.K : nullptr;
        uint32_t eq_seen = 0;
        for (int i0 = beg; i0 < end; i0 += 128) {
            const KeyBatch kb = load_keys(sj, i0, end, lane);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const bool is_gt = kb.in[u] && kb.key[u] > prefix[j];
                const bool is_eq = kb.in[u] && kb.key[u] == prefix[j];
                const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
                const bool sel = is_gt || (is_eq && eq_seen + __popc(eqm & lt_mask) < allow[j]);
                const uint32_t selm = __ballot_sync(0xffffffffu, sel);
                if (sel) {
                    const uint32_t o = out + __popc(selm & lt_mask);
                    if (o < (uint32_t)p.K) {
                        const int i = i0 + u * 32 + lane;
                        oi[o] = (int32_t)(chunk0 + i);
                        if (os) os[o] = sj[i];
                    }
                }
                out += __popc(selm);
                eq_seen += __popc(eqm);
            }
        }
    }
    named_bar_sync(1, kEpiThreads);
    return true;
}

}  // namespace dsa
