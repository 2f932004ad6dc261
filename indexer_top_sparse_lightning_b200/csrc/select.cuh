// select.cuh -- exact Top-K of shared-memory score rows, within a CTA or
// across a group of CTAs that share one sequence (sm_100a).
//
// The Top-K pass of the fused indexer ("Large Model Inference Acceleration:
// Day-0 Adaptation and Performance Optimization for New Architectures",
// section 1.1: after scoring, data stays in vector registers or shared
// memory for the weighted aggregation and the Top-K pass; no intermediate
// tensor goes to global memory).
//
// Scores are compared as order-preserving 32-bit keys (-0 folded into +0).
// The K-th largest key T is found by range histograms in key space: 2048 bins
// over [lo, hi] (bin = (key - lo) >> shift); the bin holding the K-th largest
// element is either resolved exactly from a short list of its keys or becomes
// the next, 2^11 times narrower, range.
//
// A group of G CTAs sharing one sequence meets once:
//   1. each CTA publishes the keys at or above the lower edge e_r of the bin
//      of its local c-th largest score, c = min(K, 2K/G + 32) (about twice its
//      expected share of the Top-K), with its count and e_r;
//   2. bounded group barrier;
//   3. every CTA loads all published keys into shared memory (the key stages,
//      idle by then) and finds T', the K-th largest published key.  If
//      T' >= e_r for every r, every key >= T' was published, so T = T'.
//      Otherwise (a CTA held far more than its share) the CTAs with e_r > T'
//      publish every key >= T', the group meets again, and the K-th largest
//      of the enlarged set is exact (T >= T', and all keys >= T' are in it).
//   4. per lower-ranked CTA, the published keys above / equal to T give this
//      CTA's output offset and its share of the tied elements.
// Elements above T are selected; elements equal to T are selected lowest
// position first (CTAs own contiguous position ranges in rank order, and
// within a CTA warp w owns the w-th eighth).  Indices are written in
// ascending position order with ballots and prefix counts.
#pragma once
#include "common.h"
#include "ptx.cuh"

namespace dsa {

constexpr int kBins = 2048;      // range histogram bins (11 bits)
constexpr int kListCap = 1024;   // keys of the threshold bin resolved exactly

struct SelectSmem {
    uint32_t scan[kEpiWarps];
    uint32_t kmin[4], kmax[4];   // order keys of the visible local scores, per token (from the epilogue)
    uint32_t res_bin, res_kk, res_cnt;
    uint32_t fill;               // list / published-key fill counter
    uint32_t cmin;               // smallest published key
    uint32_t wcnt[kEpiWarps][2]; // [warp][gt, eq]
    uint32_t wallow[kEpiWarps];
    uint32_t edge[4];            // this CTA's publication edge, per token
    uint32_t wpub[4][kEpiWarps]; // [token][warp] published elements
    uint32_t g_lo, g_hi, g_total, g_resident, g_max_edge;
    uint32_t gphase;             // phase of the published-key load barrier
};

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t code) {
    atomicCAS(status, 0u, code);
}

// Bounded barrier among the CTAs of one group (called by the select
// threads).  Sense-reversing: the last arriver resets the count and bumps
// the generation.  `gen` is thread 0's copy of the generation, read once per
// work item and advanced here, so a barrier costs one atomic and the wait.
// `extra` (a test hook, normally 0) makes the barrier wait for arrivals that
// never come, so that the bounded wait runs out.
static __device__ bool group_barrier(uint32_t* sync, int G, uint32_t& gen, uint32_t* status, volatile int* abort,
                              uint64_t limit_ns, uint32_t extra) {
    named_bar_sync(1, kEpiThreads);
    if (threadIdx.x == 0 && !*abort) {
        uint32_t* count = sync;
        uint32_t* genp = sync + 1;
        const uint32_t old = atom_add_acq_rel_gpu(count, 1u);
        if (old == (uint32_t)G - 1u + extra) {
            *reinterpret_cast<volatile uint32_t*>(count) = 0u;
            st_release_gpu(genp, gen + 1u);
        } else {
            const uint64_t t0 = globaltimer();
            while (ld_acquire_gpu(genp) == gen) {
                if (globaltimer() - t0 > limit_ns) {
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

// Exclusive prefix over the select threads; *total receives the sum.
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
    for (int w = 0; w < kEpiWarps; ++w) {
        const uint32_t s = scratch[w];
        if (w < warp) before += s;
        all += s;
    }
    named_bar_sync(1, kEpiThreads);
    *total = all;
    return before + x - v;
}

// The bin (of nb, higher bin = larger keys) holding the kk-th largest counted
// element, the rank of that element inside the bin and the bin's count, in
// sm->res_*.  kk must not exceed the total count.
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nb, uint32_t kk, SelectSmem* sm) {
    const int per = nb / kEpiThreads;
    const int hi_bin = nb - 1 - (int)threadIdx.x * per;
    uint32_t s = 0;
    for (int i = 0; i < per; ++i) s += hist[hi_bin - i];
    uint32_t total;
    const uint32_t before = epi_exclusive_scan(s, sm->scan, &total);
    if (before < kk && kk <= before + s) {
        uint32_t c = before;
        for (int i = 0; i < per; ++i) {
            const uint32_t h = hist[hi_bin - i];
            if (c + h >= kk) {
                sm->res_bin = (uint32_t)(hi_bin - i);
                sm->res_kk = kk - c;
                sm->res_cnt = h;
                break;
            }
            c += h;
        }
    }
    named_bar_sync(1, kEpiThreads);
}

// Histogram increment; a warp whose lanes all hit one bin (ties) adds once.
// Called by all 32 lanes of a warp.
__device__ __forceinline__ void hist_add(uint32_t* hist, bool in, uint32_t bin) {
    const uint32_t b0 = __shfl_sync(0xffffffffu, bin, 0);
    if (__all_sync(0xffffffffu, in && bin == b0)) {
        if ((threadIdx.x & 31) == 0) red_add_shared(hist + b0, 32u);
    } else if (in) {
        red_add_shared(hist + bin, 1u);
    }
}

constexpr int kU = 4;   // keys per thread and loop iteration (independent loads in flight)

// Histogram of the stream's keys in [lo, hi], bin = (key - lo) >> shift.
template <class Stream>
__device__ void stream_hist(const Stream& st, uint32_t lo, uint32_t hi, int shift, uint32_t* hist) {
    const int n = st.size();
    for (int i0 = 0; i0 < n; i0 += kEpiThreads * kU) {
        uint32_t k[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int i = i0 + u * kEpiThreads + (int)threadIdx.x;
            k[u] = i < n ? st.key(i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int i = i0 + u * kEpiThreads + (int)threadIdx.x;
            hist_add(hist, i < n && k[u] >= lo && k[u] <= hi, (k[u] - lo) >> shift);
        }
    }
}

// Appends the stream's keys in [lo, hi] to dst (any order); sm->fill counts them.
template <class Stream, class Sink>
__device__ void stream_collect(const Stream& st, uint32_t lo, uint32_t hi, uint32_t* fill, Sink sink) {
    const int n = st.size();
    const int lane = threadIdx.x & 31;
    for (int i0 = 0; i0 < n; i0 += kEpiThreads * kU) {
        uint32_t k[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int i = i0 + u * kEpiThreads + (int)threadIdx.x;
            k[u] = i < n ? st.key(i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int i = i0 + u * kEpiThreads + (int)threadIdx.x;
            const bool in = i < n && k[u] >= lo && k[u] <= hi;
            const uint32_t m = __ballot_sync(0xffffffffu, in);
            uint32_t at = 0;
            if (lane == 0 && m) at = atom_add_shared(fill, (uint32_t)__popc(m));
            at = __shfl_sync(0xffffffffu, at, 0);
            if (in) sink(at + __popc(m & ((1u << lane) - 1u)), k[u]);
        }
    }
}

// Right shift that maps [lo, hi] onto at most kBins bins.
__device__ __forceinline__ int range_shift(uint32_t lo, uint32_t hi) {
    const int bits = 32 - __clz(hi - lo);        // hi - lo < 2^bits
    return bits > 11 ? bits - 11 : 0;
}

// Streams of keys with a flat index: this CTA's scores (shared memory floats),
// published keys loaded into shared memory (ranks padded to 4 with key 0,
// which no score maps to), or the same read in place from global memory.
struct ScoreStream {
    const float* s;
    int n;
    __device__ __forceinline__ int size() const { return n; }
    __device__ __forceinline__ uint32_t key(int i) const { return order_key(s[i]); }
};
struct SmemKeyStream {
    const uint32_t* k;
    int n;
    __device__ __forceinline__ int size() const { return n; }
    __device__ __forceinline__ uint32_t key(int i) const { return k[i]; }
};
struct GlobalKeyStream {
    const uint32_t* rt;        // shared rank table [G] {count, flat offset}
    const uint32_t* cand;      // slot of rank 0
    int64_t slot;              // keys between the slots of consecutive ranks
    int G, n;
    mutable int cur = 0;       // rank of this thread's last index (indices mostly increase)
    __device__ __forceinline__ int size() const { return n; }
    __device__ uint32_t key(int i) const {
        if ((int)rt[2 * cur + 1] > i) cur = 0;
        while (cur + 1 < G && (int)rt[2 * (cur + 1) + 1] <= i) ++cur;
        const uint32_t e = (uint32_t)i - rt[2 * cur + 1];
        return e < rt[2 * cur] ? __ldcg(cand + cur * slot + e) : 0u;
    }
};

// Exact kk-th largest key among the n keys in `list`.  Short lists (at most
// 256): every element counts the larger and equal ones (broadcast reads, one
// barrier); longer ones: radix select with 8-bit digits in hist[0..255].
static __device__ uint32_t list_select(const uint32_t* list, int n, uint32_t kk, uint32_t* hist, SelectSmem* sm) {
    static_assert(2 * kEpiThreads >= 256, "short lists: at most two elements per thread");
    if (n <= 256) {
        uint32_t mine[2];
        uint32_t gt[2] = {0u, 0u}, eq[2] = {0u, 0u};
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = (int)threadIdx.x + u * kEpiThreads;
            mine[u] = i < n ? list[i] : 0u;
        }
        for (int i = 0; i < n; ++i) {
            const uint32_t x = list[i];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                gt[u] += x > mine[u];
                eq[u] += x == mine[u];
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = (int)threadIdx.x + u * kEpiThreads;
            if (i < n && gt[u] < kk && kk <= gt[u] + eq[u]) sm->res_bin = mine[u];   // equal keys write one value
        }
        named_bar_sync(1, kEpiThreads);
        const uint32_t T = sm->res_bin;
        named_bar_sync(1, kEpiThreads);
        return T;
    }
    uint32_t prefix = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += kEpiThreads) hist[i] = 0u;
        named_bar_sync(1, kEpiThreads);
        const uint32_t hmask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
        for (int i0 = 0; i0 < n; i0 += kEpiThreads) {
            const int i = i0 + (int)threadIdx.x;
            const uint32_t key = i < n ? list[i] : 0u;
            const bool in = i < n && (key & hmask) == (prefix & hmask);
            hist_add(hist, in, (key >> shift) & 255u);
        }
        named_bar_sync(1, kEpiThreads);
        find_bin(hist, 256, kk, sm);
        prefix |= sm->res_bin << shift;
        kk = sm->res_kk;
    }
    return prefix;
}

// The kk-th largest key of the stream among its keys in [lo, hi] (kk no more
// than their count): range histograms, then the exact step on the short list
// of the final bin.
template <class Stream>
__device__ uint32_t find_threshold(const Stream& st, uint32_t lo, uint32_t hi, uint32_t kk, uint32_t* hist,
                                   uint32_t* list, SelectSmem* sm, bool first_hist_ready = false) {
    while (lo != hi) {
        const int shift = range_shift(lo, hi);
        if (!first_hist_ready) {
            for (int i = threadIdx.x; i < kBins; i += kEpiThreads) hist[i] = 0u;
            named_bar_sync(1, kEpiThreads);
            stream_hist(st, lo, hi, shift, hist);
            named_bar_sync(1, kEpiThreads);
        }
        first_hist_ready = false;
        find_bin(hist, kBins, kk, sm);
        const uint32_t b = sm->res_bin, cnt = sm->res_cnt;
        kk = sm->res_kk;
        const uint32_t blo = lo + (b << shift);
        if (shift == 0) return blo;                       // the bin is one key
        const uint32_t bhi = min(hi, blo + ((1u << shift) - 1u));
        if (cnt <= (uint32_t)kListCap) {
            if (threadIdx.x == 0) sm->fill = 0u;
            named_bar_sync(1, kEpiThreads);
            stream_collect(st, blo, bhi, &sm->fill, [&](uint32_t at, uint32_t key) { list[at] = key; });
            named_bar_sync(1, kEpiThreads);
            return list_select(list, (int)cnt, kk, hist, sm);
        }
        lo = blo;
        hi = bhi;
    }
    return lo;
}

// The kk-th largest key of a long stream whose keys span [lo, hi].  A strided
// sample of 512 keys brackets it: the sample ranks kk*S/n -/+ (4 sigma + 4)
// give a window [wlo, whi]; one pass counts the keys above the window and
// histograms those inside it.  If the kk-th largest lies inside (above < kk
// <= above + inside), the search goes on in the window with kk - above;
// otherwise over the whole range.  Either way the result is exact.
template <class Stream>
__device__ uint32_t sampled_threshold(const Stream& st, uint32_t lo, uint32_t hi, uint32_t kk, uint32_t* hist,
                                      uint32_t* list, SelectSmem* sm) {
    constexpr int S = 4 * kEpiThreads;
    const int n = st.size();
    if (n < 8 * S || lo == hi) return find_threshold(st, lo, hi, kk, hist, list, sm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int step = n / S;
    const int shift = range_shift(lo, hi);
    for (int i = threadIdx.x; i < kBins; i += kEpiThreads) hist[i] = 0u;
    named_bar_sync(1, kEpiThreads);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint32_t key = st.key(((int)threadIdx.x + u * kEpiThreads) * step);
        hist_add(hist, true, (key - lo) >> shift);
    }
    named_bar_sync(1, kEpiThreads);
    const float r = (float)kk * (float)S / (float)n;
    const float pr = r / (float)S;
    const float slack = 4.0f * sqrtf((float)S * pr * (1.0f - pr)) + 4.0f;
    const uint32_t r_hi = (uint32_t)fmaxf(1.0f, floorf(r - slack));
    const uint32_t r_lo = (uint32_t)fminf((float)S, ceilf(r + slack));
    find_bin(hist, kBins, r_hi, sm);
    const uint32_t b_hi = sm->res_bin;
    find_bin(hist, kBins, r_lo, sm);
    const uint32_t b_lo = sm->res_bin;
    const uint32_t wlo = lo + (b_lo << shift);
    const uint32_t whi = min(hi, lo + (b_hi << shift) + ((1u << shift) - 1u));
    const int wshift = range_shift(wlo, whi);
    for (int i = threadIdx.x; i < kBins; i += kEpiThreads) hist[i] = 0u;
    named_bar_sync(1, kEpiThreads);
    uint32_t above = 0, inside = 0;
    for (int i0 = 0; i0 < n; i0 += kEpiThreads * kU) {
        uint32_t k[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int i = i0 + u * kEpiThreads + (int)threadIdx.x;
            k[u] = i < n ? st.key(i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int i = i0 + u * kEpiThreads + (int)threadIdx.x;
            const bool in = i < n && k[u] >= wlo && k[u] <= whi;
            above += (i < n && k[u] > whi);
            inside += in;
            hist_add(hist, in, (k[u] - wlo) >> wshift);
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        above += __shfl_xor_sync(0xffffffffu, above, o);
        inside += __shfl_xor_sync(0xffffffffu, inside, o);
    }
    if (lane == 0) {
        sm->wcnt[warp][0] = above;
        sm->wcnt[warp][1] = inside;
    }
    named_bar_sync(1, kEpiThreads);
    above = inside = 0;
#pragma unroll
    for (int w = 0; w < kEpiWarps; ++w) {
        above += sm->wcnt[w][0];
        inside += sm->wcnt[w][1];
    }
    named_bar_sync(1, kEpiThreads);
    if (above < kk && kk <= above + inside)
        return find_threshold(st, wlo, whi, kk - above, hist, list, sm, true);
    return find_threshold(st, lo, hi, kk, hist, list, sm);
}

struct GroupView {
    uint32_t* sync;     // {count, gen}
    uint32_t* hdr;      // [ranks][NQ][4]: published count, smallest published key, largest key, edge
    uint32_t* cand;     // published keys: slot of the group's first CTA
    int G, rank;
};

// Exact Top-K of NQ tokens' score rows held in shared memory (s_score, token
// j at j*stride, nloc[j] valid entries starting at position chunk0).
// Writes out_idx/out_score rows [t0 + j] in ascending position order.
// Called by the select threads; sm->kmin/kmax[j] hold the smallest and
// largest key of the visible scores.  s_hist holds kBins words, s_list
// kListCap; `scratch` (scratch_bytes, 16-byte aligned) is shared memory that
// is free in grouped work (the key stages).
template <int NQ>
__device__ bool topk_select(const IndexerParams& p, const GroupView& gv, uint32_t& gen, float* s_score,
                            int stride, const int (&nloc)[NQ], const bool (&active)[NQ], int64_t chunk0,
                            int64_t t0, uint32_t* s_hist, uint32_t* s_list, uint8_t* scratch, int scratch_bytes,
                            SelectSmem* sm, volatile int* abort, uint64_t wlim, uint32_t inject, uint64_t* gbar) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const uint32_t K = (uint32_t)p.K;
    const int G = gv.G;
    const int64_t slot_keys = p.cand_slot / NQ;

    // warp w owns the w-th eighth of a token's elements (eighths are multiples of 32)
    int qlen[NQ], list_off[NQ];
    int list_words = 0;     // u16 entries of all per-warp lists
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
        qlen[j] = ((nloc[j] + kEpiWarps * 32 - 1) / (kEpiWarps * 32)) * 32;
        list_off[j] = list_words;
        list_words += kEpiWarps * qlen[j];
    }
    // Grouped work keeps, per warp, the position-ordered list of its published
    // elements (a superset of its selected ones) when the lists take at most
    // half of the scratch; otherwise its whole eighth is scanned again.
    const int list_bytes = ((list_words * 2 + 15) / 16) * 16;
    const bool lists = G > 1 && 2 * list_bytes <= scratch_bytes;
    uint16_t* s_lists = reinterpret_cast<uint16_t*>(scratch);
    uint8_t* gscratch = scratch + (lists ? list_bytes : 0);
    const int gscratch_bytes = scratch_bytes - (lists ? list_bytes : 0);

    // The n-th element of warp `warp`'s sequence for token j: in list mode the
    // listed local indices, otherwise its eighth.
    auto seq_len = [&](int j) -> int {
        if (lists) return (int)sm->wpub[j][warp];
        const int beg = warp * qlen[j];
        return max(0, min(nloc[j], beg + qlen[j]) - beg);
    };
    auto seq_idx = [&](int j, int t) -> int {
        return lists ? (int)s_lists[list_off[j] + warp * qlen[j] + t] : warp * qlen[j] + t;
    };

    // ---- publication (grouped work)
    auto my_slot = [&](int j) { return gv.cand + (int64_t)gv.rank * p.cand_slot + j * slot_keys; };
    // per-warp counts (and lists) of the elements with key >= edge
    auto build = [&](int j, uint32_t edge) {
        const float* sj = s_score + j * stride;
        const int beg = warp * qlen[j];
        const int end = min(nloc[j], beg + qlen[j]);
        uint16_t* lw = s_lists + list_off[j] + warp * qlen[j];
        uint32_t n = 0;
        for (int i0 = beg; i0 < end; i0 += 32 * kU) {
            uint32_t k[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int i = i0 + u * 32 + lane;
                k[u] = i < end ? order_key(sj[i]) : 0u;
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int i = i0 + u * 32 + lane;
                const bool in = i < end && k[u] >= edge;
                const uint32_t m = __ballot_sync(0xffffffffu, in);
                if (lists && in) lw[n + __popc(m & lt_mask)] = (uint16_t)i;
                n += __popc(m);
            }
        }
        if (lane == 0) sm->wpub[j][warp] = n;
    };
    // rank table and (if they fit) all published keys of token j in shared memory
    uint32_t* rt = reinterpret_cast<uint32_t*>(gscratch);
    uint32_t* keys = rt + ((2 * G + 3) & ~3);
    const int keys_cap = (gscratch_bytes - ((2 * G + 3) & ~3) * 4) / 4;   // u32 keys that fit after the rank table

    // publish token j's elements >= edge (after build): keys in warp order, padded with
    // zero keys to a multiple of four (the readers' bulk loads move whole 16-byte
    // units), then the header.  The keys are staged in shared memory and leave with
    // one bulk store (small global stores from this CTA are slow next to a copy
    // engine transfer); if they do not fit there, they are stored directly.
    auto publish = [&](int j, uint32_t edge) {
        build(j, edge);
        if (threadIdx.x == 0) sm->cmin = 0xFFFFFFFFu;
        named_bar_sync(1, kEpiThreads);
        const float* sj = s_score + j * stride;
        uint32_t off = 0, tot = 0;
#pragma unroll
        for (int w = 0; w < kEpiWarps; ++w) {
            if (w < warp) off += sm->wpub[j][w];
            tot += sm->wpub[j][w];
        }
        const uint32_t tot_pad = (tot + 3u) & ~3u;
        const bool staged = (int)tot_pad <= keys_cap;
        uint32_t* slot = staged ? keys + off : my_slot(j) + off;
        if (staged) {
            fence_proxy_async_smem();   // the scratch last held copy-engine data
            for (uint32_t i = tot + threadIdx.x; i < tot_pad; i += kEpiThreads) keys[i] = 0u;
        } else {
            for (uint32_t i = tot + threadIdx.x; i < tot_pad; i += kEpiThreads) __stcg(my_slot(j) + i, 0u);
        }
        uint32_t kmn = 0xFFFFFFFFu;
        if (lists) {
            const uint16_t* lw = s_lists + list_off[j] + warp * qlen[j];
            const int n = (int)sm->wpub[j][warp];
            for (int q0 = 0; q0 < n; q0 += 32 * kU) {
                uint32_t k[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int t = q0 + u * 32 + lane;
                    k[u] = t < n ? order_key(sj[lw[t]]) : 0xFFFFFFFFu;
                }
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int t = q0 + u * 32 + lane;
                    if (t < n) {
                        if (staged) slot[t] = k[u];
                        else __stcg(slot + t, k[u]);
                    }
                    kmn = min(kmn, k[u]);
                }
            }
        } else {
            const int beg = warp * qlen[j];
            const int end = min(nloc[j], beg + qlen[j]);
            uint32_t o = 0;
            for (int i0 = beg; i0 < end; i0 += 32) {
                const int i = i0 + lane;
                const uint32_t key = i < end ? order_key(sj[i]) : 0u;
                const bool in = i < end && key >= edge;
                const uint32_t m = __ballot_sync(0xffffffffu, in);
                if (in) {
                    if (staged) slot[o + __popc(m & lt_mask)] = key;
                    else __stcg(slot + o + __popc(m & lt_mask), key);
                    kmn = min(kmn, key);
                }
                o += __popc(m);
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) kmn = min(kmn, __shfl_xor_sync(0xffffffffu, kmn, o));
        if (lane == 0) red_min_shared(&sm->cmin, kmn);
        named_bar_sync(1, kEpiThreads);
        if (threadIdx.x == 0) {
            if (staged && tot_pad > 0) {
                fence_proxy_async_smem();   // the staged keys -> the copy engine
                bulk_store(my_slot(j), keys, tot_pad * 4u);
                bulk_store_wait();          // written before the group is told (barrier below)
            }
            __threadfence();
            sm->edge[j] = edge;
            uint32_t* h = gv.hdr + ((int64_t)gv.rank * NQ + j) * 4;
            __stcg(reinterpret_cast<uint4*>(h), make_uint4(tot, sm->cmin, sm->kmax[j], edge));
        }
        named_bar_sync(1, kEpiThreads);
    };

    auto gather = [&](int j) {
        // headers of ranks tid + u * threads (G <= 256), read together; flat offsets
        // of the (4-padded) ranks by a prefix over rank order
        constexpr int HS = 256 / kEpiThreads;
        static_assert(HS * kEpiThreads == 256, "header slots per thread cover 256 ranks");
        uint4 h[HS];
#pragma unroll
        for (int u = 0; u < HS; ++u) {
            const int r = (int)threadIdx.x + u * kEpiThreads;
            h[u] = r < G ? __ldcg(reinterpret_cast<const uint4*>(gv.hdr + ((int64_t)r * NQ + j) * 4))
                         : make_uint4(0u, 0xFFFFFFFFu, 0u, 0u);
        }
        if (threadIdx.x == 0) {
            sm->g_lo = 0xFFFFFFFFu;
            sm->g_hi = 0u;
            sm->g_max_edge = 0u;
        }
        uint32_t offs[HS], totall = 0;
#pragma unroll
        for (int u = 0; u < HS; ++u) {
            uint32_t tu;
            offs[u] = totall + epi_exclusive_scan((h[u].x + 3u) & ~3u, sm->scan, &tu);
            totall += tu;
        }
        uint32_t lo = 0xFFFFFFFFu, hi = 0u, emax = 0u;
#pragma unroll
        for (int u = 0; u < HS; ++u) {
            const int r = (int)threadIdx.x + u * kEpiThreads;
            if (r < G) {
                rt[2 * r] = h[u].x;
                rt[2 * r + 1] = offs[u];
                if (h[u].x) {
                    lo = min(lo, h[u].y);
                    hi = max(hi, h[u].z);
                }
                emax = max(emax, h[u].w);
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
            emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
        }
        if ((threadIdx.x & 31) == 0) {
            red_min_shared(&sm->g_lo, lo);
            red_max_shared(&sm->g_hi, hi);
            red_max_shared(&sm->g_max_edge, emax);
        }
        if (threadIdx.x == 0) {
            const uint32_t off = totall;
            sm->g_total = off;
            sm->g_resident = (int64_t)((2 * G + 3) & ~3) * 4 + (int64_t)off * 4 <= (int64_t)gscratch_bytes;
        }
        named_bar_sync(1, kEpiThreads);
        if (sm->g_resident) {
            // every rank's (padded) keys by one bulk load each, counted on an mbarrier,
            // then the first range histogram of the threshold search
            const uint32_t glo = sm->g_lo, ghi = sm->g_hi;
            const int shift0 = glo < ghi ? range_shift(glo, ghi) : 0;
            for (int i = threadIdx.x; i < kBins; i += kEpiThreads) s_hist[i] = 0u;
            const uint32_t ph = sm->gphase;
            if (warp == 0) {
                // the scratch was last read by these threads and written by copy engines
                fence_proxy_async_smem();
                if (lane == 0) mbar_arrive_expect_tx(gbar, sm->g_total * 4u);
                __syncwarp();
                for (int r = lane; r < G; r += 32) {
                    const uint32_t n4 = (rt[2 * r] + 3u) & ~3u;
                    if (n4) bulk_load(keys + rt[2 * r + 1], gv.cand + (int64_t)r * p.cand_slot + j * slot_keys, n4 * 4u, gbar);
                }
            }
            const bool landed = mbar_wait(gbar, ph, abort, wlim);
            named_bar_sync(1, kEpiThreads);
            if (threadIdx.x == 0) sm->gphase = ph ^ 1u;
            if (!landed) *abort = 1;
            const int n = (int)sm->g_total;
            for (int i0 = 0; i0 < n; i0 += kEpiThreads * kU) {
                uint32_t k[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int i = i0 + u * kEpiThreads + (int)threadIdx.x;
                    k[u] = i < n ? keys[i] : 0u;
                }
                // padding keys 0 are below glo and not counted
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int i = i0 + u * kEpiThreads + (int)threadIdx.x;
                    hist_add(s_hist, i < n && k[u] >= glo && k[u] <= ghi, (k[u] - glo) >> shift0);
                }
            }
            named_bar_sync(1, kEpiThreads);
        }
    };
    auto group_T = [&](int j) -> uint32_t {
        if (sm->g_resident)
            return find_threshold(SmemKeyStream{keys, (int)sm->g_total}, sm->g_lo, sm->g_hi, K, s_hist, s_list, sm,
                                  true);
        return find_threshold(GlobalKeyStream{rt, gv.cand + j * slot_keys, p.cand_slot, G, (int)sm->g_total},
                              sm->g_lo, sm->g_hi, K, s_hist, s_list, sm);
    };

    if (G > 1) {
        // ---- 1. publish: the keys at or above an estimate of the local c-th
        // largest, c about twice this CTA's expected share of the Top-K: the
        // matching rank (with 25% slack) of a strided sample of 512 scores,
        // read off a range histogram of the sample -- the lower edge of its
        // bin.  A low estimate only costs the second round.
        const uint32_t c = min(K, 2u * K / (uint32_t)G + 32u);
#pragma unroll
        for (int j = 0; j < NQ; ++j) {
            if (!active[j]) continue;
            uint32_t edge = 0u;      // publish every key
            const uint32_t lo = sm->kmin[j], hi = sm->kmax[j];
            if (nloc[j] > (int)c && lo != hi) {
                const float* sj = s_score + j * stride;
                const int S = min(nloc[j], 4 * kEpiThreads);
                const int step = nloc[j] / S;
                const int shift = range_shift(lo, hi);
                for (int i = threadIdx.x; i < kBins; i += kEpiThreads) s_hist[i] = 0u;
                named_bar_sync(1, kEpiThreads);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = (int)threadIdx.x + u * kEpiThreads;
                    const uint32_t key = i < S ? order_key(sj[i * step]) : 0u;
                    hist_add(s_hist, i < S, (key - lo) >> shift);
                }
                named_bar_sync(1, kEpiThreads);
                // the sample rank matching 1.25 c of nloc, plus two
                const uint64_t want = ((uint64_t)c * 5u * (uint64_t)S + 4u * (uint64_t)nloc[j] - 1u) /
                                          (4u * (uint64_t)nloc[j]) + 2u;
                find_bin(s_hist, kBins, want < (uint64_t)S ? (uint32_t)want : (uint32_t)S, sm);
                edge = lo + (sm->res_bin << shift);
            }
            publish(j, edge);
        }
        if (!group_barrier(gv.sync, G, gen, p.status, abort, wlim, inject & 1u)) return false;
    }

#pragma unroll
    for (int j = 0; j < NQ; ++j) {
        if (!active[j]) continue;
        const float* sj = s_score + j * stride;
        uint32_t T, take = 0, base = 0;
        if (G == 1) {
            // ---- exact threshold over this CTA's own scores
            T = sampled_threshold(ScoreStream{sj, nloc[j]}, sm->kmin[j], sm->kmax[j], K, s_hist, s_list, sm);
        } else {
            // ---- 2. threshold over the published keys
            gather(j);
            T = group_T(j);
            if (sm->g_max_edge > T) {
                // some CTA held more than it published (every CTA sees the same
                // keys, so all take this branch): once every CTA has read the
                // first publication, the CTAs whose edge is above T publish all
                // their keys >= T, and the threshold of the enlarged set is exact
                const uint32_t t1 = T;
                if (!group_barrier(gv.sync, G, gen, p.status, abort, wlim, inject & 1u)) return false;
                if (sm->edge[j] > t1) publish(j, t1);
                if (!group_barrier(gv.sync, G, gen, p.status, abort, wlim, inject & 1u)) return false;
                gather(j);
                T = group_T(j);
            }
            // ---- 3. published keys above / equal to T: all ranks, and ranks below this
            // one -- the ranks lie in rank order in the flat key index, so "below" is
            // the prefix [0, offset of this rank)
            uint32_t gt_b = 0, eq_b = 0, gt_all = 0;
            const uint32_t mine = rt[2 * gv.rank + 1];
            auto count = [&](const auto& st) {
                const int n = st.size();
                for (int i0 = 0; i0 < n; i0 += kEpiThreads * kU) {
                    uint32_t k[kU];
#pragma unroll
                    for (int u = 0; u < kU; ++u) {
                        const int i = i0 + u * kEpiThreads + (int)threadIdx.x;
                        k[u] = i < n ? st.key(i) : 0u;
                    }
#pragma unroll
                    for (int u = 0; u < kU; ++u) {
                        const uint32_t i = (uint32_t)(i0 + u * kEpiThreads + (int)threadIdx.x);
                        const bool low = i < mine;
                        gt_all += k[u] > T;
                        gt_b += low && k[u] > T;
                        eq_b += low && k[u] == T;
                    }
                }
            };
            if (sm->g_resident) count(SmemKeyStream{keys, (int)sm->g_total});
            else count(GlobalKeyStream{rt, gv.cand + j * slot_keys, p.cand_slot, G, (int)sm->g_total});
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                gt_b += __shfl_xor_sync(0xffffffffu, gt_b, o);
                eq_b += __shfl_xor_sync(0xffffffffu, eq_b, o);
                gt_all += __shfl_xor_sync(0xffffffffu, gt_all, o);
            }
            if (lane == 0) {
                sm->wcnt[warp][0] = gt_b;
                sm->wcnt[warp][1] = eq_b;
                sm->wallow[warp] = gt_all;
            }
            named_bar_sync(1, kEpiThreads);
            uint32_t gtb = 0, eqb = 0, gta = 0;
#pragma unroll
            for (int w = 0; w < kEpiWarps; ++w) {
                gtb += sm->wcnt[w][0];
                eqb += sm->wcnt[w][1];
                gta += sm->wallow[w];
            }
            named_bar_sync(1, kEpiThreads);
            // K - (keys above T) tied keys are taken, lowest ranks first
            const uint32_t need_eq = K - gta;
            base = gtb + min(need_eq, eqb);
            take = need_eq > eqb ? need_eq - eqb : 0u;
        }

        // ---- per-warp counts of this CTA's elements above / equal to T, over
        // the warp's position-ordered sequence (list or eighth)
        // (float compares against T's value: the same order as the keys for
        // finite scores, and -0 == +0 like the folded keys)
        const int n = seq_len(j);
        const float Tf = key_to_float(T);
        uint32_t gt = 0, eq = 0;
        for (int q0 = 0; q0 < n; q0 += 32 * kU) {
            float f[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int t = q0 + u * 32 + lane;
                f[u] = t < n ? sj[seq_idx(j, t)] : -__int_as_float(0x7f800000);
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                gt += f[u] > Tf;
                eq += f[u] == Tf;
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            gt += __shfl_xor_sync(0xffffffffu, gt, o);
            eq += __shfl_xor_sync(0xffffffffu, eq, o);
        }
        if (lane == 0) {
            sm->wcnt[warp][0] = gt;
            sm->wcnt[warp][1] = eq;
        }
        named_bar_sync(1, kEpiThreads);
        uint32_t gt_before = 0, eq_before = 0, cgt = 0, ceq = 0, weq = 0;
#pragma unroll
        for (int w = 0; w < kEpiWarps; ++w) {
            const uint32_t g = sm->wcnt[w][0], e = sm->wcnt[w][1];
            if (w < warp) {
                gt_before += g;
                eq_before += e;
            }
            if (w == warp) weq = e;
            cgt += g;
            ceq += e;
        }
        if (G == 1) take = K - cgt;          // this CTA holds every element
        take = min(take, ceq);
        // ---- this warp's share of the tied elements, output offsets
        const uint32_t allow = take > eq_before ? min(take - eq_before, weq) : 0u;
        named_bar_sync(1, kEpiThreads);
        if (lane == 0) sm->wallow[warp] = allow;
        named_bar_sync(1, kEpiThreads);
        // ---- emission in ascending position order
        uint32_t out = base + gt_before;
        for (int w = 0; w < warp; ++w) out += sm->wallow[w];
        int32_t* oi = p.out_idx + (t0 + j) * p.K;
        float* os = p.out_score ? p.out_score + (t0 + j) * p.K : nullptr;
        uint32_t eq_seen = 0;
        for (int q0 = 0; q0 < n; q0 += 32 * kU) {
            float f[kU];
            int ix[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int t = q0 + u * 32 + lane;
                ix[u] = t < n ? seq_idx(j, t) : 0;
                f[u] = t < n ? sj[ix[u]] : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int t = q0 + u * 32 + lane;
                const bool is_gt = t < n && f[u] > Tf;
                const bool is_eq = t < n && f[u] == Tf;
                const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
                const bool sel = is_gt || (is_eq && eq_seen + __popc(eqm & lt_mask) < allow);
                const uint32_t selm = __ballot_sync(0xffffffffu, sel);
                if (sel) {
                    const uint32_t o = out + __popc(selm & lt_mask);
                    if (o < K) {
                        oi[o] = (int32_t)(chunk0 + ix[u]);
                        if (os) os[o] = f[u];
                    }
                }
                out += __popc(selm);
                eq_seen += __popc(eqm);
            }
        }
        named_bar_sync(1, kEpiThreads);
    }
    return true;
}

}  // namespace dsa
