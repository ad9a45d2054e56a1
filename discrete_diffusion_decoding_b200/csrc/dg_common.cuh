// Shared definitions of the CUDA library: the Philox generator, the workspace
// layout and the schedule that maps (position tile, vocabulary block) work onto
// groups of CTAs of the fused kernel.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/dg.h"

namespace dg {

constexpr int kCanvas = 256;      // positions per canvas
constexpr int kTileM = 128;       // positions per tile (UMMA M)
constexpr int kBV = 256;          // vocabulary rows per logits tile (UMMA N)
constexpr int kKChunk = 128;      // hidden columns per pipeline stage of the logits GEMM
constexpr int kVChunk = 128;      // vocabulary rows per pipeline stage of the self-conditioning GEMM
constexpr int kMaxSlice = 256;    // widest self-conditioning column slice a CTA pair keeps in TMEM
constexpr int kMaxCanvas = 256;   // canvases per call (the fused kernel keeps the active list in shared memory)
constexpr int kMaxParts = 64;     // vocabulary shards one dg_denoise_merge call takes
constexpr int kThreads = 256;     // threads of the fused kernel
// The fused kernel's operand rings: every pipeline stage is one A box (h rows or P^T
// columns, both read from L2) and one B box (W rows or E columns, mostly from DRAM), each
// 32 KB per CTA; the B ring is one stage deeper so that more of the DRAM-bound operand is
// in flight.
#ifndef DG_A_STAGES
#define DG_A_STAGES 3
#endif
#ifndef DG_B_STAGES
#define DG_B_STAGES 4
#endif
constexpr int kAStages = DG_A_STAGES;
constexpr int kBStages = DG_B_STAGES;
constexpr int kRingBoxBytes = 32 * 1024;
// With E aliasing W, this many tenths of the hidden columns of every W tile keep normal
// L2 priority between the logits and the self-conditioning pass (the rest is streamed).
#ifndef DG_KEEP_W_TENTHS
#define DG_KEEP_W_TENTHS 3
#endif
constexpr int kKeepWTenths = DG_KEEP_W_TENTHS;
constexpr int kFusedSmemBytes = (kAStages + kBStages) * kRingBoxBytes + 1024 + 4 * kMaxCanvas;
constexpr float kLazyRescale = 8.0f;  // log2 units the shared reference may lag the running max

// ------------------------------------------------------------------ Philox4x32-10
// Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11):
// ten rounds; per round the two 32x32->64 products of counter words 0 and 2 with
// the multipliers, the high halves xored with the other words and the key; the key
// advances by the Weyl increments between rounds.
__host__ __device__ inline void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
    for (int r = 0; r < 10; ++r) {
        if (r) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c[0];
        const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c[2];
        const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c[1] ^ k0;
        const uint32_t n1 = static_cast<uint32_t>(p1);
        const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c[3] ^ k1;
        const uint32_t n3 = static_cast<uint32_t>(p0);
        c[0] = n0;
        c[1] = n1;
        c[2] = n2;
        c[3] = n3;
    }
}

// floor(word0 * V / 2^32) for counter (i, s, c, tag) under the canvas seed.
__host__ __device__ inline int32_t philox_token(uint64_t seed, uint32_t i, uint32_t s, uint32_t c, uint32_t tag,
                                                uint32_t vocab) {
    uint32_t ctr[4] = {i, s, c, tag};
    philox4x32_10(ctr, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
    return static_cast<int32_t>((static_cast<uint64_t>(ctr[0]) * vocab) >> 32);
}

enum : uint32_t { kTagInit = 0, kTagRenoise = 1, kTagStubTarget = 2, kTagStubNoise = 3 };
// sampled acceptance: counter (v / 64, step, canvas, kTagSample + 256 i), one per 64-entry chunk
constexpr uint32_t kTagSample = 4;

// ------------------------------------------------------------------ tile-major head layout
// Element (v, c) of a [V, d] head stored tile-major: atoms of 128 rows x 64 columns, ordered
// by row tile then column atom, each atom row-major (64 contiguous columns per row).
__host__ __device__ inline size_t tiled_index(long long v, int c, int d) {
    return (static_cast<size_t>(v >> 7) * (d >> 6) + (c >> 6)) * 8192 + static_cast<size_t>(v & 127) * 64 + (c & 63);
}

// ------------------------------------------------------------------ plan and layout
struct Plan {
    int C, N, V, d;
    int group;        // G: CTA pairs sharing one logits tile stream, each pair owning d/G columns
    int slice;        // d / G
    int n_groups;     // groups resident at once (grid = n_groups * G pairs = 2 n_groups G CTAs)
    int steps_per_tile;  // vocabulary blocks of G * kBV rows per canvas
    int max_seg;      // partial slots per group
    int n_slots;      // n_groups * max_seg
    int fp8;          // E4M3 logits operands (the workspace then holds the quantised hidden states)
    int tiled;        // W and E in the tile-major head layout (tiled_index)
};

struct Layout {
    size_t prev_argmax, stable, stop, err;        // per-canvas state
    size_t clk;                                   // [4] uint64: SM cycles and global ns at the start
                                                  // and end of CTA 0's MMA loop (last fused pass)
    size_t counters;                              // [n_groups][4] uint32, 128 B apart
    size_t rowmax;                                // [n_groups][2][G][256] float
    size_t pbuf;                                  // [n_groups][2][G][kBV vocab][256 rows] bf16 (P^T)
    size_t stats;                                 // [n_slots][G][256] float4 {m, l, u, best}
    size_t stat_idx;                              // [n_slots][G][256] int32
    size_t skey;                                  // [n_slots][G][256] float: best Gumbel-max key (sampled mode)
    size_t sidx;                                  // [n_slots][G][256] int32: its vocabulary index
    size_t kept;                                  // [N] int32: token an accepted position keeps (group rule)
    size_t opart;                                 // [n_slots][256][d] float
    size_t hq, hexp;                              // E4M3 logits: [N][d] codes and [N] exponents of h
    size_t total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline Layout make_layout(const Plan& pl) {
    Layout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o = align_up(o + bytes, 256);
        return at;
    };
    L.prev_argmax = take(sizeof(int32_t) * pl.N);
    L.stable = take(sizeof(int32_t) * pl.C);
    L.stop = take(sizeof(int32_t) * pl.C);
    L.err = take(sizeof(int32_t) * 4);
    L.clk = take(sizeof(unsigned long long) * 4);
    L.counters = take(static_cast<size_t>(128) * 4 * pl.n_groups);
    L.rowmax = take(sizeof(float) * pl.n_groups * 2 * pl.group * kCanvas);
    L.pbuf = take(static_cast<size_t>(2) * pl.n_groups * 2 * pl.group * kCanvas * kBV);
    L.stats = take(sizeof(float) * 4 * static_cast<size_t>(pl.n_slots) * pl.group * kCanvas);
    L.stat_idx = take(sizeof(int32_t) * static_cast<size_t>(pl.n_slots) * pl.group * kCanvas);
    L.skey = take(sizeof(float) * static_cast<size_t>(pl.n_slots) * pl.group * kCanvas);
    L.sidx = take(sizeof(int32_t) * static_cast<size_t>(pl.n_slots) * pl.group * kCanvas);
    L.kept = take(sizeof(int32_t) * pl.N);
    L.opart = take(sizeof(float) * static_cast<size_t>(pl.n_slots) * kCanvas * pl.d);
    if (pl.fp8) {
        L.hq = take(static_cast<size_t>(pl.N) * pl.d);
        L.hexp = take(sizeof(int32_t) * static_cast<size_t>(pl.N));
    }
    L.total = o;
    return L;
}

// Work schedule of the fused kernel.  Each position tile's vocabulary blocks are
// split into k contiguous ranges; the n_pt * k pieces are numbered range-major
// (pi = j * n_pt + pt) and dealt round-robin to the groups (group pi % n_groups,
// round pi / n_groups).  Groups working in the same round therefore stream the
// same vocabulary rows for different tiles at the same time, so the rows are
// fetched from DRAM once and shared through L2, and every group gets the same
// number of pieces.  k = n_groups / gcd(n_pt, n_groups) balances exactly; when
// that would give a group more than kMaxPieces pieces, whole tiles are dealt
// instead (k = 1).
constexpr int kMaxPieces = 64;

__host__ __device__ inline int ranges_per_tile(int n_pt, int n_groups) {
    int a = n_pt, b = n_groups;
    while (b) {
        const int t = a % b;
        a = b;
        b = t;
    }
    const int k = n_groups / a;
    return (static_cast<long long>(n_pt) * k + n_groups - 1) / n_groups > kMaxPieces ? 1 : k;
}

__host__ __device__ inline int pieces_per_group(int n_pt, int n_groups) {
    const int k = ranges_per_tile(n_pt, n_groups);
    return static_cast<int>((static_cast<long long>(n_pt) * k + n_groups - 1) / n_groups);
}

// Piece of group g in round j: its position tile and block range [tb, te) (possibly empty).
__host__ __device__ inline bool piece_of(int g, int j, int n_groups, int n_pt, int T, int& pt, int& tb, int& te) {
    const int k = ranges_per_tile(n_pt, n_groups);
    const long long pi = static_cast<long long>(j) * n_groups + g;
    if (pi >= static_cast<long long>(n_pt) * k) return false;
    const int jj = static_cast<int>(pi / n_pt);
    pt = static_cast<int>(pi % n_pt);
    tb = static_cast<int>(static_cast<long long>(jj) * T / k);
    te = static_cast<int>(static_cast<long long>(jj + 1) * T / k);
    return te > tb;
}

// Offsets of the four per-group counters (uint32 words).
enum : int { kCntRowmax = 0, kCntP = 1, kCntUsed = 2 };
__host__ __device__ inline size_t counter_word(int g, int which) { return static_cast<size_t>(g) * 128 + which * 32; }

}  // namespace dg
