// common.h -- parameter blocks and shared-memory layouts shared by the host
// launcher (api.cu) and the kernels.  No arithmetic of the method lives here.
#pragma once
#include <cstddef>
#include <cstdint>

namespace dsa {

constexpr int kPage = 64;             // tokens per cache page
constexpr int kTileKeys = 128;        // keys per indexer MMA tile (two pages)
constexpr int kMaxTopK = 2048;
constexpr int kDqk = 576;             // latent 512 + RoPE 64
constexpr int kDv = 512;
constexpr int kEpiWarps = 8;          // indexer epilogue / Top-K warps (two per TMEM lane quarter)
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kConvThreads = 192;     // fp8 key widening threads (six warps)

// Device status word values (mirrors dsa_status).
enum : uint32_t {
    kStOk = 0, kStTimeout = 5, kStBounds = 6, kStCapacity = 7
};

// Workspace header (first 256 bytes).
struct WsHeader {
    uint32_t status;
    uint32_t pad[63];
};

// ------------------------------------------------------------------ indexer
// Work decomposition:
//  mode 0 (grouped): one group per query window of the launch range
//    [w_begin, w_end).  A window is up to NQ consecutive query tokens of one
//    sequence (a sequence with nq_b tokens has ceil(nq_b / NQ) windows, in
//    token order; with seq_windows every sequence is exactly one window).  A
//    window's keys are the positions its last token sees.  Each group gets g
//    CTAs, each CTA scores a contiguous chunk of key tiles, and the group
//    agrees on its Top-K through published candidate keys.
//  mode 1 (independent): every query token is its own group with one CTA;
//    CTAs loop over tokens in zig-zag order (head-tail pairing).
struct IndexerParams {
    const int32_t* seq_lens;
    const int32_t* cu_q;
    const int32_t* block_table;
    const float* w;
    const float* k_scale;     // fp8 keys: [nblk, 64, D_I/64] fp32
    const uint8_t* k_scale_e8;  // MXFP8 keys: [nblk, 64, D_I/32] shared exponents (2^(e-127))
    const uint8_t* q_codes;   // MXFP8 queries: [T, H_I, D_I] e4m3 codes
    const uint8_t* q_scale;   // MXFP8 queries: [T, H_I, D_I/32] shared exponents
    int32_t* out_idx;
    float* out_score;
    uint32_t* status;
    uint8_t* group_ws;        // mode 0: per-group sync + publication headers
    int64_t group_ws_stride;  // bytes per group
    uint32_t* cand;           // mode 0: published keys, cand_slot per CTA
    int64_t cand_slot;        // keys per CTA slot (NQ tokens share it equally)
    int32_t B, T, max_blocks, num_blocks;
    int32_t w_begin, w_end;   // mode 0 launch range (window indices)
    int32_t seq_windows;      // mode 0: every sequence has at most NQ tokens (window index = sequence)
    int32_t t_begin, t_end;   // mode 1 token range
    int32_t mode;
    int32_t K;
    int32_t score_cap;        // fp32 score slots per CTA (all tokens of a group)
};

// Group workspace layout (mode 0), per group:
//   [0,128)   sync {count, gen}
//   hdr[max_ctas][NQ][4] u32: published key count, smallest published key,
//             largest visible key, publication edge
__host__ __device__ constexpr int64_t group_ws_bytes(int nq, int max_ctas) {
    return 128 + (int64_t)max_ctas * nq * 4 * 4;
}

// Published-key slot per CTA (keys; larger than any CTA's score capacity).
constexpr int64_t kCandSlotKeys = 65536;

template <int DI, bool FP8>
struct KeyTileBytes {
    static constexpr int value = kTileKeys * DI * (FP8 ? 1 : 2);
};

// ------------------------------------------------------------------ sparse attention
struct SfaParams {
    const int32_t* seq_lens;
    const int32_t* cu_q;
    const int32_t* block_table;
    const uint16_t* kv;       // [num_blocks*64, 576] bf16 bits
    const int32_t* idx;       // [T, K]
    uint16_t* out;            // [T, H, 512] bf16 bits
    float* lse;               // [T, H] or null
    uint8_t* part;            // partials of tokens shared by several pairs: [pairs][2 sides][2 CTAs] slots
    uint32_t* status;         // status word; words 1-2 of the same area hold the test hooks
    int32_t B, T, H, K, max_blocks, num_blocks;
    int32_t early_q;          // Q may be loaded before the preceding launch completes
    int32_t align_tokens;     // pairs take whole tokens (ranges start at token boundaries)
    float scale_log2;         // sm_scale * log2(e)
};

}  // namespace dsa
