// Fused denoise-sampling pass (logits, online softmax statistics, entropy,
// argmax and self-conditioning) and the split-vocabulary combine.
//
// Method (juhoplayground "DiffusionGemma", inference mechanism: logits for
// every canvas position, temperature sharpening, self-conditioning with the
// probability-weighted token embedding; marrrang deep dive, reverse-diffusion
// steps 3-5 and the entropy criteria):
//   z = h W^T / T;  p = softmax(z);  H = LSE - sum p z;  a = argmax z;  sc = p E.
//
// Work decomposition (sm_100a, persistent grid of CTA pairs, one CTA per SM):
//  * A CTA pair (cluster of 2, cta_group::2 UMMA) owns one 256-position canvas:
//    CTA p holds positions [128p, 128p+128) (UMMA M = 256 split across the pair).
//  * A group of G pairs streams the vocabulary in blocks of G x 256 rows.  In a
//    block, pair r computes the 256 x 256 logits tile of vocabulary sub-tile r over
//    the full hidden width (each CTA loads its own h rows and half of the 256 W
//    rows; TMA -> SMEM -> tcgen05.mma -> TMEM), and owns columns
//    [r d/G, (r+1) d/G) of the self-conditioning accumulator O (fp32, TMEM).
//  * The CTAs of a group agree on a per-row reference maximum for the block (row
//    maxima exchanged through L2 with release/acquire counters), so every CTA
//    turns its logits into P = 2^(z log2e - m_ref) in bf16 against the same
//    reference, publishes P to an L2-resident scratch tile, and the pair
//    accumulates O[:, slice] += P_q E[q-rows, slice] for all G tiles q of the
//    block (second pair UMMA, E as an MN-major operand split by columns).  The
//    reference only moves when the running maximum exceeds it by 8 (log2 units),
//    and then O is rescaled in TMEM.
//  * Each CTA keeps exact per-row partial statistics of its own tiles relative
//    to the shared reference: l = sum e, u = sum e (z - m_ref), and the best raw
//    logit with its smallest vocabulary index.  The sampled-acceptance instance
//    (dg_fused_sample_kernel) also keeps, per row, the best Gumbel-max key of the
//    64-entry chunks' log-masses and the entry drawn inside the leading chunk.
//  * Streamed operands carry an L2 evict-first policy; when E aliases W the
//    first 3/10 of every W tile's hidden-column stages keep normal priority so
//    that the self-conditioning GEMM re-reads them from L2.
//  * Work is dealt in pieces (a range of blocks of one canvas) so that groups in
//    the same round stream the same vocabulary rows for different canvases (rows
//    come from DRAM once and are shared through L2); each piece ends with O and
//    the statistics written as a partial, merged by dg_combine_kernel.
//
// Roles inside a CTA (256 threads): warp 0 issues the A operand's TMA loads
// (h, or P^T) into a ring of 3 x 32 KB stages and warp 3 the B operand's (W, or
// E) into a ring of 4 x 32 KB stages (both CTAs of a pair load; completion is
// counted on the leader's barriers); warp 1 allocates TMEM and, in the leader
// CTA, issues the pair UMMAs; warps 4-7 (one TMEM lane quarter each, thread =
// position row) do the softmax, publish P^T and run the epilogue.  Every wait is
// bounded (see dg_sm100.cuh); the producers leave only once every load they
// issued into either CTA has landed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "dg_common.cuh"
#include "dg_fused.h"
#include "dg_sm100.cuh"

namespace dg {

namespace {

constexpr int kBox = kRingBoxBytes;              // one A or B box per CTA per stage
constexpr uint32_t kAtomCol = 128u * 128u;     // bytes of one 64-column swizzle atom column of a 128-row box
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0;             // logits tile columns [0, 256)
constexpr uint32_t kTmemO = 256;           // self-conditioning slice columns [256, 256 + slice)
constexpr int kSoftmaxWarp0 = 4;
constexpr int kMaxSlotsPerTile = 256;      // >= ranges per tile (at most the group count)

// error codes recorded in the workspace error word
enum : int {
    kErrProducerEmpty = 101, kErrProducerP = 102, kErrProducerDrain = 103,
    kErrMmaFull = 201, kErrMmaSFree = 202, kErrMmaOReady = 203, kErrMmaDrain = 204,
    kErrSmaxSFull = 301, kErrSmaxRowmax = 302, kErrSmaxUsed = 303, kErrSmaxODone = 304,
};

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded poll until *ctr >= target (wrap-safe comparison): the waits on other CTAs of
// the group, limited by limit_ns (a kernel argument; the waits that drain this CTA's
// own loads and UMMAs keep the fixed DG_WAIT_LIMIT_NS).
__device__ bool wait_counter(const uint32_t* ctr, uint32_t target, volatile int* abort, int* err, int code,
                             uint64_t limit_ns) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        if (static_cast<int32_t>(ld_acquire_u32(ctr) - target) >= 0) return true;
        if (*abort) return false;
        if ((it & 15u) == 0) {
            const uint64_t now = global_ns();
            if (it == 0) {
                t0 = now;
            } else if (now - t0 > limit_ns) {
                atomicCAS(err, 0, code);
                raise_pair_abort(abort);
                return false;
            }
        }
        __nanosleep(32);
    }
}

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// 2^x on the SFU (documented PTX ex2.approx; relative error about 2^-22, 2^-inf = +0).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log2(x) on the SFU (documented PTX lg2.approx; relative error about 2^-22).
__device__ __forceinline__ float fast_log2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 64 consecutive TMEM columns of this thread's lane, two loads in flight per wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&v)[64]) {
    uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
    uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
    tmem_ld32(taddr, lo);
    tmem_ld32(taddr + 32, hi);
    tmem_wait_ld();
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    uint32_t a[16], b[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        a[i] = r[i];
        b[i] = r[16 + i];
    }
    tmem_st16(taddr, a);
    tmem_st16(taddr + 16, b);
}

// The pieces of one group, in round order (see piece_of).
struct Schedule {
    int g, n_groups, n_ct, T, nseg;
    __device__ void init(int g_, int n_groups_, int n_ct_, int steps_per_tile) {
        g = g_;
        n_groups = n_groups_;
        n_ct = n_ct_;
        T = steps_per_tile;
        nseg = n_ct > 0 ? pieces_per_group(n_ct, n_groups) : 0;
    }
    // false for an empty piece (every role skips it the same way)
    __device__ bool seg(int j, int& ct, int& tb, int& te) const {
        return piece_of(g, j, n_groups, n_ct, T, ct, tb, te);
    }
};

}  // namespace

// -log2(u) for u = (w + 1/2) 2^-32, from eps = 1 - u = (~w + 1/2) 2^-32: the SFU
// logarithm of 1 - eps, or below eps = 2^-8 the series log2(e) (eps + eps^2/2 + eps^3/3)
// (relative truncation error < 2^-26), which keeps full precision as u -> 1.  Then
// -log2(-log2 u) is the standard Gumbel variable g = -ln(-ln u) in log2 units, up to
// the constant log2(log2 e).
__device__ __forceinline__ float neg_log2_uniform(uint32_t w) {
    const float eps = fmaf(static_cast<float>(~w), 2.3283064365386963e-10f, 1.1641532182693481e-10f);
    const float series = eps * fmaf(eps, fmaf(eps, 0.333333343f, 0.5f), 1.0f) * 1.44269502f;
    return eps < 0.00390625f ? series : -fast_log2(1.0f - eps);
}

template <bool kSample, bool kFp8>
__device__ __forceinline__ void fused_pass(const FusedArgs& a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* a_ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* b_ring = a_ring + kAStages * kBox;
    int* active = reinterpret_cast<int*>(b_ring + kBStages * kBox);

    // a_* / b_*: the A and B rings' barriers (full: the leader's, counting both CTAs' bytes)
    __shared__ uint64_t a_full[kAStages], a_empty[kAStages], b_full[kBStages], b_empty[kBStages];
    __shared__ uint64_t s_full, s_free, o_ready, o_done, drain_bar;
    // producer drain: per side and ring slot, 1 + the index of the last use issued into it
    // (0: none) and that use's bytes for one CTA (both CTAs load boxes of the same size);
    // own_* this CTA's, peer_* (leader CTA) the peer's
    __shared__ uint32_t own_use[2][kBStages], own_bytes[2][kBStages];
    __shared__ uint32_t peer_use[2][kBStages], peer_bytes[2][kBStages];
    __shared__ uint64_t peer_bar[2];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    __shared__ int n_active_s;
    __shared__ int rescale_any;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int G = a.G;
    const uint32_t prank = cluster_ctarank();        // 0 = pair leader (issues the UMMAs)
    const bool leader = prank == 0;
    const int pair = blockIdx.x >> 1;
    const int g = pair / G;
    const int r = pair % G;
    const int d0 = r * a.slice;

    if (tid == 0) {
        for (int i = 0; i < kAStages; ++i) {
            mbar_init(&a_full[i], 1);        // leader: one expect_tx arrival per use, bytes of both CTAs
            mbar_init(&a_empty[i], 1);       // one multicast commit per use
        }
        for (int i = 0; i < kBStages; ++i) {
            mbar_init(&b_full[i], 1);
            mbar_init(&b_empty[i], 1);
        }
        mbar_init(&s_full, 1);
        mbar_init(&s_free, 2);               // leader: softmax of both CTAs
        mbar_init(&o_ready, 2);              // leader: softmax of both CTAs
        mbar_init(&o_done, 1);
        mbar_init(&drain_bar, 1);
        mbar_init(&peer_bar[0], 1);          // one remote arrival from the peer's producer of each side
        mbar_init(&peer_bar[1], 1);
        for (int i = 0; i < 2 * kBStages; ++i) {
            own_use[i / kBStages][i % kBStages] = 0;
            own_bytes[i / kBStages][i % kBStages] = 0;
        }
        fence_mbar_init_cluster();
        abort_flag = 0;
        rescale_any = 0;
    }
    if (warp == 2) {
        // active canvases in increasing order
        int base = 0;
        for (int c0 = 0; c0 < a.C; c0 += 32) {
            const int c = c0 + lane;
            const bool act = c < a.C && a.stop[c] == 0;
            const uint32_t m = __ballot_sync(0xffffffffu, act);
            if (act) active[base + __popc(m & ((1u << lane) - 1u))] = c;
            base += __popc(m);
        }
        if (lane == 0) n_active_s = base;
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();        // barriers of both CTAs initialised before any remote arrival
    tc_fence_after();

    const uint32_t tmem = tmem_base;
    Schedule sch;
    sch.init(g, a.n_groups, n_active_s, a.steps_per_tile);
    auto sub_valid = [&](int t, int q) { return static_cast<long long>(t * G + q) * kBV < a.V; };
    auto vocab0 = [&](int t, int q) { return (t * G + q) * kBV; };

    uint32_t* cnt_rowmax = a.counters + counter_word(g, kCntRowmax);
    uint32_t* cnt_p = a.counters + counter_word(g, kCntP);
    uint32_t* cnt_used = a.counters + counter_word(g, kCntUsed);
    // logits stages per W tile: 256 bytes of each row per stage (128 bf16 or 256 E4M3 values)
    const int n_sstages = kFp8 ? a.d / 256 : a.d / kKChunk;
    const int n_ech = a.slice / 128;                 // E atoms (64 columns each) per CTA per O stage
    const uint32_t e_box_bytes = static_cast<uint32_t>(n_ech) * kAtomCol;   // <= kBox (slice <= 256)
    const int nG2 = 2 * G;                           // CTAs per group

    if (warp == 0 || warp == 3) {
        // ===================================================== TMA producers (both CTAs)
        // Warp 0 issues the A operand of every stage (h rows, or the P^T columns of
        // this CTA's positions) and posts the stage's expected bytes on the leader's
        // barrier; warp 3 issues the B operand (this CTA's half of the W rows, or of
        // the E columns).  Two issuers keep more loads in flight than one.
        if (lane == 0) {
            const bool a_side = warp == 0;
            tma_prefetch_desc(a_side ? &a.map_h : &a.map_w);
            tma_prefetch_desc(a_side ? &a.map_p : &a.map_e);
            // L2 policy: E rows are dead once the self-conditioning pass has read them, and so
            // are W rows unless E aliases W; with aliasing, the first keep_w_stages column
            // stages of every W tile keep normal priority (the two blocks in flight of every
            // group would not fit in L2 whole) and are read again from L2 as E
            const uint64_t pol_stream = l2_policy_evict_first();
            // this side's ring: its stage count, buffers and barriers
            const int n_st = a_side ? kAStages : kBStages;
            uint8_t* my_ring = a_side ? a_ring : b_ring;
            uint64_t* my_full = a_side ? a_full : b_full;
            uint64_t* my_empty = a_side ? a_empty : b_empty;
            auto full_leader = [&](int slot) { return smem_addr_in_rank(&my_full[slot], 0); };
            uint32_t it = 0;
            bool ok = true;
            const int side = a_side ? 0 : 1;
            uint32_t* last_use = own_use[side];
            uint32_t* last_bytes = own_bytes[side];
            auto acquire = [&](int& slot) -> bool {
                slot = static_cast<int>(it % n_st);
                if (it >= static_cast<uint32_t>(n_st) &&
                    !mbar_wait(&my_empty[slot], ((it / n_st) - 1) & 1, &abort_flag, a.err, kErrProducerEmpty))
                    return false;
                ++it;
                return true;
            };
            // a use of `slot` whose load brings `bytes` into each CTA of the pair; the leader
            // posts both CTAs' bytes on its barrier
            auto arm = [&](int slot, uint32_t bytes) {
                last_use[slot] = it;
                last_bytes[slot] = bytes;
                if (leader) mbar_arrive_expect_tx(&my_full[slot], 2u * bytes);
            };
            auto emit_o = [&](int k, int t) -> bool {
                if (a_side) {
                    if (!wait_counter(cnt_p, static_cast<uint32_t>(nG2 * (k + 1)), &abort_flag, a.err, kErrProducerP,
                                      a.counter_wait_ns))
                        return false;
                    fence_async_global();
                }
                for (int q = 0; q < G; ++q) {
                    if (!sub_valid(t, q)) continue;
                    // P^T tile of (block k, sub-tile q): [256 vocab rows][256 canvas rows]
                    const int prow = ((g * 2 + (k & 1)) * G + q) * kBV;
                    for (int vc = 0; vc < kBV / kVChunk; ++vc) {
                        int slot;
                        if (!acquire(slot)) return false;
                        uint8_t* st = my_ring + slot * kBox;
                        if (a_side) {
                            arm(slot, 2u * kAtomCol);
                            // both 64-row atoms of this CTA's canvas rows in one 3-D box
                            tma_load_3d_pair(st, &a.map_p, full_leader(slot), 0, prow + vc * kVChunk,
                                             static_cast<int>(prank) * 2);
                        } else {
                            arm(slot, e_box_bytes);
                            // this CTA's half of the column slice (n_ech atoms of 64 columns) in one 3-D box
                            const int er = vocab0(t, q) + vc * kVChunk;
                            const int ec = (d0 + static_cast<int>(prank) * (a.slice / 2)) / 64;
                            if (a.tiled)      // tile (er / 128, ec): n_ech consecutive atoms, one contiguous block
                                tma_load_3d_pair_hint(st, &a.map_e, full_leader(slot), 0, 0,
                                                      (er >> 7) * (a.d >> 6) + ec, pol_stream);
                            else
                                tma_load_3d_pair_hint(st, &a.map_e, full_leader(slot), 0, er, ec, pol_stream);
                        }
                    }
                }
                return true;
            };
            int k = 0;
            for (int j = 0; j < sch.nseg && ok; ++j) {
                int ct, tb, te;
                if (!sch.seg(j, ct, tb, te)) continue;
                const int row0 = active[ct] * kCanvas + static_cast<int>(prank) * kTileM;
                for (int t = tb; t < te && ok; ++t, ++k) {
                    if (sub_valid(t, r)) {
                        const int v0 = vocab0(t, r) + static_cast<int>(prank) * (kBV / 2);
                        for (int kc = 0; kc < n_sstages; ++kc) {
                            int slot;
                            if (!acquire(slot)) { ok = false; break; }
                            uint8_t* st = my_ring + slot * kBox;
                            arm(slot, kBox);
                            if (a_side) {
                                tma_load_3d_pair(st, &a.map_h, full_leader(slot), 0, row0, kc * (kKChunk / 64));
                            } else {
                                // row-major: box at rows v0, column block kc * 2; tiled: the two atoms of
                                // tile (v0 / 128, kc * 2), one contiguous 32 KB block
                                const int wy = a.tiled ? 0 : v0;
                                const int wz = a.tiled ? (v0 >> 7) * (a.d >> 6) + kc * 2 : kc * (kKChunk / 64);
                                if (kc < a.keep_w_stages)
                                    tma_load_3d_pair(st, &a.map_w, full_leader(slot), 0, wy, wz);
                                else
                                    tma_load_3d_pair_hint(st, &a.map_w, full_leader(slot), 0, wy, wz, pol_stream);
                            }
                        }
                    }
                    if (ok && t > tb) ok = emit_o(k - 1, t - 1);
                }
                if (ok) ok = emit_o(k - 1, te - 1);
            }
            // drain: every load issued into either CTA of the pair has landed before the
            // pair passes its last cluster barrier.  All loads complete on the leader's full
            // barriers, so the peer hands its last use of every slot to the leader, and the
            // leader waits for the last phase of every slot.  A producer issues use u + n_st
            // of a slot only after use u was consumed, which needs both CTAs' bytes; so after
            // an abort the two CTAs' last uses of a slot differ by at most one round, and the
            // leader settles that round: bytes the peer never sent are completed here, and a
            // use only the peer issued is armed here with the peer's bytes.
            if (!leader) {
                for (int sl = 0; sl < n_st; ++sl) {
                    st_shared_rank_u32(&peer_use[side][sl], 0, last_use[sl]);
                    st_shared_rank_u32(&peer_bytes[side][sl], 0, last_bytes[sl]);
                }
                mbar_arrive_remote(&peer_bar[side], 0);      // release: the stores above first
            } else {
                auto drain_wait = [&](uint64_t* bar, uint32_t parity, bool cluster) -> bool {
                    const uint32_t ba = smem_u32(bar);
                    const uint64_t t0 = global_ns();
                    while (!(cluster ? mbar_try_wait_cluster(ba, parity) : mbar_try_wait(ba, parity))) {
                        if (global_ns() - t0 > DG_WAIT_LIMIT_NS) {
                            atomicCAS(a.err, 0, kErrProducerDrain);
                            return false;
                        }
                    }
                    return true;
                };
                if (drain_wait(&peer_bar[side], 0, true)) {
                    for (int sl = 0; sl < n_st; ++sl) {
                        const uint32_t ul = last_use[sl], un = peer_use[side][sl];
                        if (ul == 0 && un == 0) continue;
                        if (ul > un)
                            mbar_complete_tx(&my_full[sl], last_bytes[sl]);
                        else if (un > ul)
                            mbar_arrive_expect_tx(&my_full[sl], peer_bytes[side][sl]);
                        const uint32_t u = (ul > un ? ul : un) - 1;
                        if (!drain_wait(&my_full[sl], (u / n_st) & 1, false)) break;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ===================================================== pair UMMA issuer (leader CTA)
        if (lane == 0 && leader) {
            const uint32_t idesc_s =
                kFp8 ? idesc_e4m3_f32(2 * kTileM, kBV, false, false) : idesc_bf16_f32(2 * kTileM, kBV, false, false);
            const uint32_t idesc_o = idesc_bf16_f32(2 * kTileM, a.slice, true, true);
            uint32_t it = 0;
            bool ok = true;
            // stage `it`: A box in A-ring slot it % kAStages, B box in B-ring slot it % kBStages
            int sa = 0, sb = 0;
            auto consume = [&](uint32_t& a_addr, uint32_t& b_addr) -> bool {
                sa = static_cast<int>(it % kAStages);
                sb = static_cast<int>(it % kBStages);
                if (!mbar_wait(&a_full[sa], (it / kAStages) & 1, &abort_flag, a.err, kErrMmaFull)) return false;
                if (!mbar_wait(&b_full[sb], (it / kBStages) & 1, &abort_flag, a.err, kErrMmaFull)) return false;
                ++it;
                tc_fence_after();
                a_addr = smem_u32(a_ring + sa * kBox);
                b_addr = smem_u32(b_ring + sb * kBox);
                return true;
            };
            auto release = [&]() {
                umma_commit_pair(&a_empty[sa], 0x3);
                umma_commit_pair(&b_empty[sb], 0x3);
            };
            // seg_first: block t is the first of its piece, so O starts from zero
            auto do_o = [&](int k, int t, bool seg_first) -> bool {
                if (!mbar_wait(&o_ready, k & 1, &abort_flag, a.err, kErrMmaOReady)) return false;
                tc_fence_after();
                bool first = seg_first;
                for (int q = 0; q < G; ++q) {
                    if (!sub_valid(t, q)) continue;
                    for (int vc = 0; vc < kBV / kVChunk; ++vc) {
                        uint32_t sta, stb;
                        if (!consume(sta, stb)) return false;
#pragma unroll
                        for (int kk = 0; kk < kVChunk / 16; ++kk) {
                            const uint64_t ad = smem_desc(sta + kk * 2048, kAtomCol, 1024, kSwizzle128B);
                            const uint64_t bd = smem_desc(stb + kk * 2048, kAtomCol, 1024, kSwizzle128B);
                            umma_ss_pair(tmem + kTmemO, ad, bd, idesc_o, (first && kk == 0) ? 0u : 1u);
                        }
                        first = false;
                        release();
                    }
                }
                // every P tile of block k has landed in both CTAs' shared memory
                red_release_add(cnt_used, 1u);
                umma_commit_pair(&o_done, 0x3);
                return true;
            };
            int k = 0;
            // the SM clock this pass runs at: cycles and global time over CTA 0's issue loop
            const unsigned long long clk0 = clock64(), ns0 = global_ns();
            for (int j = 0; j < sch.nseg && ok; ++j) {
                int ct, tb, te;
                if (!sch.seg(j, ct, tb, te)) continue;
                for (int t = tb; t < te && ok; ++t, ++k) {
                    if (k > 0 && !mbar_wait(&s_free, (k - 1) & 1, &abort_flag, a.err, kErrMmaSFree)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (sub_valid(t, r)) {
                        for (int kc = 0; kc < n_sstages; ++kc) {
                            uint32_t sta, stb;
                            if (!consume(sta, stb)) { ok = false; break; }
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                // K step kk (32 bytes: 16 bf16 or 32 E4M3 values): atom column kk / 4,
                                // 32-byte offset (kk % 4) inside the swizzled 128-byte row
                                const uint32_t ko = (kk >> 2) * kAtomCol + (kk & 3) * 32;
                                const uint64_t ad = smem_desc(sta + ko, 16, 1024, kSwizzle128B);
                                const uint64_t bd = smem_desc(stb + ko, 16, 1024, kSwizzle128B);
                                if constexpr (kFp8)
                                    umma_ss_pair_f8(tmem + kTmemS, ad, bd, idesc_s, (kc | kk) != 0 ? 1u : 0u);
                                else
                                    umma_ss_pair(tmem + kTmemS, ad, bd, idesc_s, (kc | kk) != 0 ? 1u : 0u);
                            }
                            release();
                        }
                        if (!ok) break;
                        umma_commit_pair(&s_full, 0x3);
                    } else {
                        mbar_arrive_remote(&s_full, 0);
                        mbar_arrive_remote(&s_full, 1);
                    }
                    if (t > tb) ok = do_o(k - 1, t - 1, t - 1 == tb);
                }
                if (ok) ok = do_o(k - 1, te - 1, te - 1 == tb);
            }
            if (blockIdx.x == 0) {
                const unsigned long long clk1 = clock64(), ns1 = global_ns();
                a.clk[0] = clk0;
                a.clk[1] = ns0;
                a.clk[2] = clk1;
                a.clk[3] = ns1;
            }
            // drain: all issued UMMAs complete before TMEM is released
            umma_commit_pair(&drain_bar, 0x1);
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(smem_u32(&drain_bar), 0)) {
                if (global_ns() - t0 > DG_WAIT_LIMIT_NS) {
                    atomicCAS(a.err, 0, kErrMmaDrain);
                    break;
                }
            }
        }
    } else if (warp >= kSoftmaxWarp0) {
        // ===================================================== softmax / epilogue
        // Every bounded wait below is followed by a softmax-warp barrier and a
        // check of the shared abort flag, so the 128 threads always leave
        // together and never strand each other at a barrier.
        const int row = (warp - kSoftmaxWarp0) * 32 + lane;      // row within this CTA's 128
        const int crow = static_cast<int>(prank) * kTileM + row; // row within the canvas
        const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const bool sleader = (tid == kSoftmaxWarp0 * 32);
        float c2 = a.scale_log2;       // log2(e) / T times the row's operand scale (E4M3 logits)
        bool ok = true;
        int k = 0;
        for (int j = 0; j < sch.nseg && ok; ++j) {
            int ct, tb, te;
            if (!sch.seg(j, ct, tb, te)) continue;
            float m_ref = -INFINITY, l = 0.f, u = 0.f, best = -INFINITY;
            int best_idx = -1;
            if constexpr (kFp8)
                c2 = ldexpf(a.scale_log2, a.row_exp[active[ct] * kCanvas + crow] + a.w_exp);
            // sampled acceptance: Philox key of this canvas, counter word 3 of this position
            float skey = -INFINITY;
            int sidx = -1;
            uint32_t key_lo = 0, key_hi = 0, pos_word = 0, canvas = 0;
            if constexpr (kSample) {
                canvas = static_cast<uint32_t>(active[ct]);
                const uint64_t seed = a.seeds[canvas];
                key_lo = static_cast<uint32_t>(seed);
                key_hi = static_cast<uint32_t>(seed >> 32);
                pos_word = kTagSample + 256u * static_cast<uint32_t>(crow);
            }
            for (int t = tb; t < te; ++t, ++k) {
                const bool valid = sub_valid(t, r);
                mbar_wait(&s_full, k & 1, &abort_flag, a.err, kErrSmaxSFull);
                softmax_bar();
                if (abort_flag) { ok = false; break; }
                tc_fence_after();
                // --- pass 1: row maximum of the raw logits tile
                float smax = -INFINITY;
                if (valid) {
#pragma unroll 1
                    for (int c0 = 0; c0 < kBV; c0 += 64) {
                        uint32_t v[64];
                        tmem_ld64(tmem + kTmemS + lane_addr + c0, v);
#pragma unroll
                        for (int i = 0; i < 64; ++i) smax = fmaxf(smax, __uint_as_float(v[i]));
                    }
                }
                float* rm = a.rowmax + static_cast<size_t>((g * 2 + (k & 1)) * G) * kCanvas;
                rm[r * kCanvas + crow] = smax * c2;
                __threadfence();
                softmax_bar();
                if (sleader) {
                    red_release_add(cnt_rowmax, 1u);
                    const bool w = wait_counter(cnt_rowmax, static_cast<uint32_t>(nG2 * (k + 1)), &abort_flag,
                                                a.err, kErrSmaxRowmax, a.counter_wait_ns);
                    // P buffer (k & 1) was last read for block k-2
                    if (w && k >= 2)
                        wait_counter(cnt_used, static_cast<uint32_t>(G * (k - 1)), &abort_flag, a.err, kErrSmaxUsed,
                                     a.counter_wait_ns);
                }
                softmax_bar();
                if (abort_flag) { ok = false; break; }
                float M = -INFINITY;
                for (int q = 0; q < G; ++q) M = fmaxf(M, __ldcg(rm + q * kCanvas + crow));
                // --- lazy shared reference (the same decision in all CTAs holding this row)
                float alpha = 1.f;
                if (m_ref == -INFINITY || M > m_ref + kLazyRescale) {
                    if (m_ref != -INFINITY) {
                        alpha = fast_exp2(m_ref - M);
                        u = alpha * (u + (m_ref - M) * l);
                        l = alpha * l;
                    }
                    m_ref = M;
                }
                // --- pass 2: probabilities, statistics, argmax, P^T tile
                // P is published transposed ([vocab][canvas row]) so that a warp's stores
                // are contiguous: lanes 2m and 2m+1 swap one value per column pair and
                // each stores the two rows (2m, 2m+1) of one column as a bf16 pair.
                if (valid) {
                    __nv_bfloat16* pt = a.pbuf + static_cast<size_t>((g * 2 + (k & 1)) * G + r) * kBV * kCanvas;
                    const bool odd = lane & 1;
                    const int prow = crow & ~1;
                    const int v0 = vocab0(t, r) + a.vocab_offset;     // global vocabulary index of column 0
#pragma unroll 1
                    for (int c0 = 0; c0 < kBV; c0 += 64) {
                        uint32_t v[64];
                        tmem_ld64(tmem + kTmemS + lane_addr + c0, v);
                        float lc = 0.f;            // this 64-entry chunk's mass, relative to m_ref
#pragma unroll
                        for (int i = 0; i < 64; i += 2) {
                            const float s0 = __uint_as_float(v[i]), s1 = __uint_as_float(v[i + 1]);
                            if (s0 > best) { best = s0; best_idx = v0 + c0 + i; }
                            if (s1 > best) { best = s1; best_idx = v0 + c0 + i + 1; }
                            const float y0 = fmaf(s0, c2, -m_ref), y1 = fmaf(s1, c2, -m_ref);
                            const float e0 = fast_exp2(y0), e1 = fast_exp2(y1);
                            lc += e0 + e1;
                            u = fmaf(e0, y0, fmaf(e1, y1, u));
                            const float recv = __shfl_xor_sync(0xffffffffu, odd ? e0 : e1, 1);
                            const int col = c0 + i + (odd ? 1 : 0);
                            *reinterpret_cast<uint32_t*>(pt + static_cast<size_t>(col) * kCanvas + prow) =
                                pack_bf16(odd ? recv : e0, odd ? e1 : recv);
                        }
                        l += lc;
                        if constexpr (kSample) {
                            // two-level draw: the chunk's Gumbel-max key on its log-mass (word 0 of
                            // Philox counter (v / 64, step, canvas, 4 + 256 i)), absolute in log2
                            // units; strict > keeps the smallest chunk on a tie.  A chunk that takes
                            // the lead picks its entry by the inverse CDF at word 1.
                            const uint32_t q = static_cast<uint32_t>(v0 + c0) >> 6;
                            uint32_t w[4] = {q, static_cast<uint32_t>(a.step), canvas, pos_word};
                            philox4x32_10(w, key_lo, key_hi);
                            const float kq = (m_ref + fast_log2(lc)) - fast_log2(neg_log2_uniform(w[0]));
                            if (kq > skey) {
                                skey = kq;
                                const float target = fmaf(static_cast<float>(w[1]), 2.3283064365386963e-10f,
                                                          1.1641532182693481e-10f) * lc;
                                float run = 0.f;
                                int pick = -1, last = 0;
#pragma unroll
                                for (int i = 0; i < 64; ++i) {
                                    const float e = fast_exp2(fmaf(__uint_as_float(v[i]), c2, -m_ref));
                                    run += e;
                                    if (pick < 0 && run > target) pick = i;
                                    if (e > 0.f) last = i;
                                }
                                sidx = v0 + c0 + (pick >= 0 ? pick : last);
                            }
                        }
                    }
                }
                tc_fence_before();
                fence_async_global();
                __threadfence();
                if (alpha != 1.f && t > tb) rescale_any = 1;
                softmax_bar();
                const bool resc = rescale_any != 0;
                if (sleader) {
                    mbar_arrive_remote(&s_free, 0);
                    red_release_add(cnt_p, 1u);
                }
                // --- O of block k-1 must be complete before block k may accumulate (and be rescaled)
                if (t > tb) {
                    mbar_wait(&o_done, (k - 1) & 1, &abort_flag, a.err, kErrSmaxODone);
                    softmax_bar();
                    if (abort_flag) { ok = false; break; }
                    tc_fence_after();
                    if (resc) {
#pragma unroll 1
                        for (int c0 = 0; c0 < a.slice; c0 += 32) {
                            uint32_t v[32];
                            tmem_ld32(tmem + kTmemO + lane_addr + c0, v);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
                            tmem_st32(tmem + kTmemO + lane_addr + c0, v);
                        }
                        tmem_wait_st();
                    }
                    tc_fence_before();
                }
                softmax_bar();
                if (sleader) {
                    rescale_any = 0;
                    mbar_arrive_remote(&o_ready, 0);
                }
            }
            if (!ok) break;
            // --- piece epilogue: O slice and statistics become a partial
            mbar_wait(&o_done, (k - 1) & 1, &abort_flag, a.err, kErrSmaxODone);
            softmax_bar();
            if (abort_flag) { ok = false; break; }
            tc_fence_after();
            const int slot = g * a.max_seg + j;
            float* orow = a.opart + (static_cast<size_t>(slot) * kCanvas + crow) * a.d + d0;
#pragma unroll 1
            for (int c0 = 0; c0 < a.slice; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + kTmemO + lane_addr + c0, v);
                tmem_wait_ld();
                float4* dst = reinterpret_cast<float4*>(orow + c0);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                         __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            }
            const size_t si = (static_cast<size_t>(slot) * G + r) * kCanvas + crow;
            a.stats[si] = make_float4(m_ref, l, u, best);
            a.stat_idx[si] = best_idx;
            if constexpr (kSample) {
                a.skey[si] = skey;
                a.sidx[si] = sidx;
            }
            tc_fence_before();
            softmax_bar();
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();        // no CTA leaves while its peer may still signal it
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

__global__ void __launch_bounds__(kThreads, 1) dg_fused_kernel(const __grid_constant__ FusedArgs a) {
    fused_pass<false, false>(a);
}

__global__ void __launch_bounds__(kThreads, 1) dg_fused_sample_kernel(const __grid_constant__ FusedArgs a) {
    fused_pass<true, false>(a);
}

__global__ void __launch_bounds__(kThreads, 1) dg_fused_fp8_kernel(const __grid_constant__ FusedArgs a) {
    fused_pass<false, true>(a);
}

__global__ void __launch_bounds__(kThreads, 1) dg_fused_fp8_sample_kernel(const __grid_constant__ FusedArgs a) {
    fused_pass<true, true>(a);
}

// ---------------------------------------------------------------------------
// Finishing a position from its merged statistics (juhoplayground, entropy
// bounded sampler; deep dive steps 4-5):
//   H = ln L - ln2 * U / L;  LSE = ln2 * (M + log2 L);
// then keep the argmax where H <= bound (in the sampled mode the Gumbel-max
// sample), otherwise a uniform vocabulary token from Philox (tag 1, this step).
// With the group rule only the kept token is stored (dg_stop_kernel decides).
// A position whose statistics come from a pass that recorded an error is
// poisoned: H and LSE NaN, argmax -1, re-noised, never accepted.
struct Finish {
    float* entropy;
    int32_t* argmax;
    float* lse;
    int32_t* tokens;
    uint8_t* accept;
    int32_t* kept;
    const uint64_t* seeds;
    float bound;
    int step, V, accept_mode, accept_rule;
};

__device__ void finish_position(const Finish& f, int n, int c, int crow, float M, float L, float U, int bidx,
                                int sidx, bool bad) {
    const float ln2 = 0.69314718055994531f;
    float H = logf(L) - ln2 * (U / L);
    float lse = ln2 * (M + log2f(L));
    if (bad) {
        H = __int_as_float(0x7fc00000);
        lse = H;
        bidx = -1;
    }
    f.entropy[n] = H;
    f.argmax[n] = bidx;
    if (f.lse) f.lse[n] = lse;
    if (!f.tokens) return;
    const int32_t renoise = philox_token(f.seeds[c], static_cast<uint32_t>(crow), static_cast<uint32_t>(f.step),
                                         static_cast<uint32_t>(c), kTagRenoise, static_cast<uint32_t>(f.V));
    const int32_t keep = f.accept_mode == 1 ? sidx : bidx;
    if (f.accept_rule == 1) {
        f.kept[n] = bad ? renoise : keep;          // accepted by groups in dg_stop_kernel
    } else {
        const bool acc = !bad && H <= f.bound;
        f.tokens[n] = acc ? keep : renoise;
        f.accept[n] = acc ? 1 : 0;
    }
}

// ---------------------------------------------------------------------------
// Split-vocabulary combine: one CTA per (active position, block of 1024
// self-conditioning columns).  Merges the partial statistics of every (piece,
// pair) covering the position's canvas:
//   M = max m_s;  L = sum_s 2^(m_s-M) sum_r l;  U = sum_s 2^(m_s-M) (sum_r u + (m_s-M) sum_r l)
//   argmax = best raw logit, smallest index;  sc = sum_s 2^(m_s-M) O_s / L.
// The column-block-0 CTA of a position finishes it (finish_position).  In shard
// mode (a vocabulary shard of a split head) it writes the merged statistics and
// the unnormalised numerator sum_s 2^(m_s-M) O_s instead.  CTA (0, 0) also clears
// the fused kernel's group counters for its next launch.
__global__ void __launch_bounds__(256) dg_combine_kernel(const CombineArgs a) {
    griddep_wait();                         // launched after the fused pass it merges
    __shared__ float sh_w[kMaxSlotsPerTile];
    __shared__ int sh_slot[kMaxSlotsPerTile];
    __shared__ int n_slots_s;
    __shared__ float sh_L;
    __shared__ int sh_bad;
    __shared__ int sh_active_rank;
    __shared__ int sh_n_active;
    __shared__ int sh_skip;

    const int n = blockIdx.x;               // position row in [0, N)
    const int c = n / kCanvas;
    const int crow = n % kCanvas;
    const int tid = threadIdx.x;
    const bool head = blockIdx.y == 0;      // writes the per-position scalars
    if (blockIdx.x == 0 && head) {
        for (int i = tid; i < a.n_groups * 128; i += blockDim.x) a.counters[i] = 0u;
    }
    if (tid == 0) {
        sh_skip = a.stop[c] != 0;
        sh_bad = a.err != nullptr && *reinterpret_cast<const volatile int*>(a.err) != 0;
        int rank = 0, na = 0;
        for (int q = 0; q < a.C; ++q) {
            const int act = a.stop[q] == 0;
            if (q < c) rank += act;
            na += act;
        }
        sh_active_rank = rank;
        sh_n_active = na;
    }
    __syncthreads();
    if (sh_skip) return;
    const int ct = sh_active_rank;
    const int T = a.steps_per_tile;
    const bool bad = sh_bad != 0;

    if (tid < 32) {
        // warp 0: merge statistics over (slot, pair) entries.  The slots of this canvas's
        // non-empty ranges are listed in range order, 32 ranges at a time (lane = range).
        const int n_ct = sh_n_active;
        const int k = ranges_per_tile(n_ct, a.n_groups);
        int ns = 0;
        for (int j0 = 0; j0 < k; j0 += 32) {
            const int jj = j0 + tid;
            bool has = false;
            int slot = 0;
            if (jj < k) {
                const int tb = static_cast<int>(static_cast<long long>(jj) * T / k);
                const int te = static_cast<int>(static_cast<long long>(jj + 1) * T / k);
                if (te > tb) {
                    const long long pi = static_cast<long long>(jj) * n_ct + ct;
                    const int gg = static_cast<int>(pi % a.n_groups), round = static_cast<int>(pi / a.n_groups);
                    has = true;
                    slot = gg * a.max_seg + round;
                }
            }
            const uint32_t m = __ballot_sync(0xffffffffu, has);
            const int at = ns + __popc(m & ((1u << tid) - 1u));
            if (has && at < kMaxSlotsPerTile) sh_slot[at] = slot;
            ns += __popc(m);
        }
        ns = min(ns, kMaxSlotsPerTile);
        if (tid == 0) n_slots_s = ns;
        __syncwarp();
        // the group reference of each slot (every pair of a piece shares it): lanes in parallel
        float M = -INFINITY;
        for (int s = tid; s < ns; s += 32)
            M = fmaxf(M, a.stats[(static_cast<size_t>(sh_slot[s]) * a.G) * kCanvas + crow].x);
#pragma unroll
        for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float L = 0.f, Uu = 0.f, best = -INFINITY, skey = -INFINITY;
        int bidx = 0x7fffffff, sidx = 0x7fffffff;
#pragma unroll 4
        for (int e = tid; e < ns * a.G; e += 32) {
            const int s = e / a.G, rr = e % a.G;
            const size_t si = (static_cast<size_t>(sh_slot[s]) * a.G + rr) * kCanvas + crow;
            const float4 st = a.stats[si];
            const int idx = a.stat_idx[si];
            const float w = exp2f(st.x - M);
            L += w * st.y;
            Uu += w * (st.z + (st.x - M) * st.y);
            if (idx >= 0 && (st.w > best || (st.w == best && idx < bidx))) {
                best = st.w;
                bidx = idx;
            }
            if (a.accept_mode == 1) {
                const float kk = a.skey[si];
                const int ki = a.sidx[si];
                if (ki >= 0 && (kk > skey || (kk == skey && ki < sidx))) {
                    skey = kk;
                    sidx = ki;
                }
            }
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            L += __shfl_xor_sync(0xffffffffu, L, off);
            Uu += __shfl_xor_sync(0xffffffffu, Uu, off);
            const float ob = __shfl_xor_sync(0xffffffffu, best, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
            if (ob > best || (ob == best && oi < bidx)) {
                best = ob;
                bidx = oi;
            }
            const float ok = __shfl_xor_sync(0xffffffffu, skey, off);
            const int oki = __shfl_xor_sync(0xffffffffu, sidx, off);
            if (ok > skey || (ok == skey && oki < sidx)) {
                skey = ok;
                sidx = oki;
            }
        }
        if (tid == 0) {
            sh_L = L;
            if (head && a.part_stats) {
                const float nan = __int_as_float(0x7fc00000);
                a.part_stats[n] = bad ? make_float4(nan, nan, nan, nan) : make_float4(M, L, Uu, best);
                a.part_idx[n] = bad ? -1 : bidx;
                a.part_skey[n] = skey;
                a.part_sidx[n] = a.accept_mode == 1 ? sidx : -1;
            } else if (head) {
                const Finish f{a.entropy, a.argmax, a.lse, a.tokens, a.accept, a.kept, a.seeds, a.bound,
                               a.step, a.V, a.accept_mode, a.accept_rule};
                finish_position(f, n, c, crow, M, L, Uu, bidx, sidx, bad);
            }
        }
        for (int s = tid; s < ns; s += 32)
            sh_w[s] = exp2f(a.stats[(static_cast<size_t>(sh_slot[s]) * a.G) * kCanvas + crow].x - M);
    }
    __syncthreads();
    float* out = a.part_o ? a.part_o : a.selfcond;
    if (out == nullptr) return;
    const int ns = n_slots_s;
    const float scale = bad ? __int_as_float(0x7fc00000) : (a.part_o ? 1.f : 1.f / sh_L);
    const int col_end = min(a.d, static_cast<int>(blockIdx.y + 1) * kCombineCols);
    for (int col = static_cast<int>(blockIdx.y) * kCombineCols + tid * 4; col < col_end; col += blockDim.x * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int s = 0; s < ns; ++s) {
            const float4 o =
                *reinterpret_cast<const float4*>(a.opart + (static_cast<size_t>(sh_slot[s]) * kCanvas + crow) * a.d + col);
            const float w = sh_w[s];
            acc.x = fmaf(w, o.x, acc.x);
            acc.y = fmaf(w, o.y, acc.y);
            acc.z = fmaf(w, o.z, acc.z);
            acc.w = fmaf(w, o.w, acc.w);
        }
        *reinterpret_cast<float4*>(out + static_cast<size_t>(n) * a.d + col) =
            make_float4(acc.x * scale, acc.y * scale, acc.z * scale, acc.w * scale);
    }
}

// ---------------------------------------------------------------------------
// Merge of vocabulary shards (a head split by vocabulary rows over several
// devices, or several calls): the same LSE merge as the combine, over the shards'
// partials instead of the pieces of one pass.  One CTA per (active position,
// block of 1024 self-conditioning columns); warp 0 merges the statistics (one
// lane per shard), then the position is finished as in the combine.  A shard
// whose statistics are NaN (its pass recorded an error) poisons the position.
__global__ void __launch_bounds__(256) dg_merge_kernel(const MergeArgs a) {
    __shared__ float sh_w[kMaxParts];
    __shared__ float sh_L;
    __shared__ int sh_bad;
    __shared__ int sh_skip;
    const int n = blockIdx.x;
    const int c = n / kCanvas;
    const int crow = n % kCanvas;
    const int tid = threadIdx.x;
    const bool head = blockIdx.y == 0;
    if (tid == 0) sh_skip = a.stop[c] != 0;
    __syncthreads();
    if (sh_skip) return;
    auto stats_of = [&](int g) {
        return reinterpret_cast<const float4*>(a.partials + static_cast<size_t>(g) * a.part_bytes + a.off_stats)[n];
    };
    if (tid < 32) {
        float M = -INFINITY;
        bool bad = false;
        for (int g = tid; g < a.n_parts; g += 32) {
            const float m = stats_of(g).x;
            bad |= m != m;
            M = fmaxf(M, m);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        bad = __any_sync(0xffffffffu, bad);
        float L = 0.f, U = 0.f, best = -INFINITY, skey = -INFINITY;
        int bidx = 0x7fffffff, sidx = 0x7fffffff;
        for (int g = tid; g < a.n_parts; g += 32) {
            const uint8_t* base = a.partials + static_cast<size_t>(g) * a.part_bytes;
            const float4 st = stats_of(g);
            const int idx = reinterpret_cast<const int32_t*>(base + a.off_idx)[n];
            const float w = exp2f(st.x - M);
            L += w * st.y;
            U += w * (st.z + (st.x - M) * st.y);
            if (idx >= 0 && (st.w > best || (st.w == best && idx < bidx))) {
                best = st.w;
                bidx = idx;
            }
            if (a.accept_mode == 1) {
                const float kk = reinterpret_cast<const float*>(base + a.off_skey)[n];
                const int ki = reinterpret_cast<const int32_t*>(base + a.off_sidx)[n];
                if (ki >= 0 && (kk > skey || (kk == skey && ki < sidx))) {
                    skey = kk;
                    sidx = ki;
                }
            }
            sh_w[g] = w;
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            L += __shfl_xor_sync(0xffffffffu, L, off);
            U += __shfl_xor_sync(0xffffffffu, U, off);
            const float ob = __shfl_xor_sync(0xffffffffu, best, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
            if (ob > best || (ob == best && oi < bidx)) {
                best = ob;
                bidx = oi;
            }
            const float ok = __shfl_xor_sync(0xffffffffu, skey, off);
            const int oki = __shfl_xor_sync(0xffffffffu, sidx, off);
            if (ok > skey || (ok == skey && oki < sidx)) {
                skey = ok;
                sidx = oki;
            }
        }
        if (tid == 0) {
            sh_L = L;
            sh_bad = bad;
            if (head) {
                const Finish f{a.entropy, a.argmax, a.lse, a.tokens, a.accept, a.kept, a.seeds, a.bound,
                               a.step, a.V, a.accept_mode, a.accept_rule};
                finish_position(f, n, c, crow, M, L, U, bidx, sidx, bad);
            }
        }
    }
    __syncthreads();
    if (a.selfcond == nullptr) return;
    const float scale = sh_bad ? __int_as_float(0x7fc00000) : 1.f / sh_L;
    const int col_end = min(a.d, static_cast<int>(blockIdx.y + 1) * kCombineCols);
    for (int col = static_cast<int>(blockIdx.y) * kCombineCols + tid * 4; col < col_end; col += blockDim.x * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int g = 0; g < a.n_parts; ++g) {
            const float* o = reinterpret_cast<const float*>(a.partials + static_cast<size_t>(g) * a.part_bytes +
                                                            a.off_o);
            const float4 v = *reinterpret_cast<const float4*>(o + static_cast<size_t>(n) * a.d + col);
            const float w = sh_w[g];
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
        }
        *reinterpret_cast<float4*>(a.selfcond + static_cast<size_t>(n) * a.d + col) =
            make_float4(acc.x * scale, acc.y * scale, acc.z * scale, acc.w * scale);
    }
}

}  // namespace dg
