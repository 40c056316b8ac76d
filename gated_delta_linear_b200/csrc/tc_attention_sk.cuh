// tc_attention_sk.cuh -- the intra-frame attention of tc_attention.cuh (the
// same per-tile pipeline, softmax and fused inter-frame read) on a grid of at
// most one CTA per SM, with the work divided evenly over the CTAs.
//
// Source: "Technical summary: Attend Locally, Remember Linearly (ARL2)",
// gist.science/ar/paper/2605.16579, §2.1 (intra-frame softmax attention over
// the frame's tokens) and §2.2 (every token reads O_inter = Q (phi_q^T S_{N-1})).
//
// Work: a row is one 128-query tile of one (batch, head); a unit is one
// (row, 128-key tile) pair, U = rows x n units for n key tiles per row.  CTA c
// of G takes the units [c U / G, (c + 1) U / G) in row-major order: a run of
// whole rows with at most a partial row at each end.  G <= rows, so a CTA
// holds at least n units and a row is split over at most two CTAs.  For the
// 480p shape (156 rows of 13 tiles) 148 CTAs take 13 or 14 units each, instead
// of 156 CTAs of 13 units in two waves, the second nearly empty.
//
// A CTA walks its items (row segments) one after another with the pipeline of
// tc_attention.cuh; every ring and buffer counter runs on across items, so the
// next item's Q load and first score products overlap the current item's last
// tiles and epilogue.  Per item: Q is loaded once the previous item's scores
// no longer read the Q buffer; the first two score products take Q from shared
// memory, the rest from TMEM; O_inter = Q W goes to the S buffer the item's
// last tile does not use, and the next item's first tile skips to the other
// buffer (one buffer step per item boundary), so only its second tile waits
// for the epilogue to have read O_inter.  The output is stored from registers.
//
// A split row: each of its two CTAs ends its segment with O (unnormalised,
// against its own running offset m) and the row sums l.  The CTA that finishes
// first publishes them in the workspace; the second (it learns which it is
// from an atomic ticket, taken after its own record is written, or after it
// has seen the other's ticket) merges: with M = max(m1, m2),
//     out = (O1 2^(m1-M) + O2 2^(m2-M)) / (l1 2^(m1-M) + l2 2^(m2-M)) + O_inter,
// the same softmax over the whole key range, and resets the ticket.  No CTA
// waits for another.  Only the head segment (the row's first key tiles, the
// last item of its CTA) computes O_inter; it adds it to its record when it
// publishes, for a tail that merges.  The tail is the first item of its CTA,
// so the CTA's first W load (which waits for the kernel that writes W) comes
// only with its second item.
#pragma once

#include "tc_attention.cuh"

namespace hyb {
namespace tc {

namespace sk {
using attn::K0;
using attn::kKStages;
using attn::kLoadVWarp;
using attn::kLoadWarp;
using attn::kMmaWarp;
using attn::kSoftmaxThreads;
using attn::kThreads;
using attn::kVStages;
using attn::Q;
using attn::SMEM;
using attn::V0;
using attn::XCH;
using attn::XFL;
using attn::BAR;
enum { B_Q = 0, B_QFREE = 1, B_QTM = 2, B_OIDONE = 3, B_ORD = 4, B_KFULL = 5, B_KEMPTY = 8, B_VFULL = 11,
       B_VEMPTY = 14, B_SFULL = 17, B_SREAD = 19, B_PFULL = 21, B_PVDONE = 22, B_DRAIN = 23, B_REC = 24,
       B_COUNT = 25 };
// after the barriers: TMEM base, abort word, per-item flags [2], ticket words [2][2],
// the deferred-merge word
static_assert(B_COUNT * 8 + 48 <= 256, "barrier block");
// partial records of a split row, per boundary: the head's O [128][128] fp32
// (unnormalised), m [128], l [128] (whole-row sums), a valid word, O_inter
// [128][128]; then the tail's O, m, l and valid word (no O_inter).  A
// [128][128] matrix is stored as float4 f = column / 4 of row r at f * 128 + r,
// so the 32 rows of a warp read or write 512 contiguous bytes at a time.
constexpr int kRecM = 128 * 128, kRecL = kRecM + 128, kRecOk = kRecL + 128, kRecOI = kRecOk + 64;
constexpr int kHeadFloats = kRecOI + 128 * 128;
constexpr int kTailFloats = kRecOk + 64;
constexpr int kSlotFloats = kHeadFloats + kTailFloats;  // a multiple of 64 floats (256 bytes)
constexpr uint32_t kTailBytes = kTailFloats * 4;        // one bulk copy into the free K and V rings
static_assert(kTailBytes % 16 == 0 && kTailBytes <= 2 * kKStages * kTileBytes, "tail record copy");
static_assert(kSlotFloats % 64 == 0, "record alignment");
constexpr int kMaxGrid = kNumSMs;

// The units of CTA c: items (row segments) and their place in the CTA's
// sequence of key tiles.
struct Work {
    long long u0, u1;
    int n, first_row, j0_first, nitems;
    __device__ void init(long long U, int G, int c, int n_) {
        n = n_;
        u0 = (long long)c * U / G;
        u1 = (long long)(c + 1) * U / G;
        first_row = (int)(u0 / n);
        j0_first = (int)(u0 - (long long)first_row * n);
        nitems = (int)((u1 - 1) / n) - first_row + 1;
    }
    __device__ int row(int ii) const { return first_row + ii; }
    __device__ int j0(int ii) const { return ii == 0 ? j0_first : 0; }
    __device__ int j1(int ii) const { return ii == nitems - 1 ? (int)(u1 - (long long)(first_row + ii) * n) : n; }
    __device__ int len(int ii) const { return j1(ii) - j0(ii); }
    // index of the item's first tile in the CTA's tile sequence
    __device__ int gbase(int ii) const { return ii == 0 ? 0 : (n - j0_first) + (ii - 1) * n; }
    // a first item that starts mid-row (the tail of a split row) has no O_inter
    // (so O_inter products, and their barrier's phases, are counted from item 1)
    __device__ bool has_oi(int ii) const { return !(ii == 0 && j0_first > 0); }
    // position of the item's first K tile in the K ring's sequence (an item with
    // O_inter also passes W_hi and W_lo through the ring after its K tiles)
    __device__ int kbase(int ii) const { return gbase(ii) + 2 * ii - (ii > 0 && j0_first > 0 ? 2 : 0); }
    __device__ int total() const { return (int)(u1 - u0); }
};
}  // namespace sk

__global__ void __launch_bounds__(sk::kThreads, 1)
    attention_sk_kernel(const __grid_constant__ LayerArgs a, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_o) {
    using namespace sk;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicOr(a.flags, FLAG_INTERNAL);
        return;
    }
    // the delta update of this pass reads nothing this kernel writes
    pdl_launch_dependents();
    const uint32_t sb = smem_u32(smem);
    uint64_t* bars = (uint64_t*)(smem + BAR);
    uint32_t* tmem_slot = (uint32_t*)(bars + B_COUNT);
    volatile int* abort_word = (volatile int*)(tmem_slot + 1);
    volatile int* item_bad = (volatile int*)(tmem_slot + 2);  // [2], by item parity
    volatile int* ticket = (volatile int*)(tmem_slot + 4);    // [2][2], by item parity: peek, ticket

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T;
    const int nqt = (T + kTile - 1) / kTile;
    const int rows = a.B * a.H * nqt;
    Work W;
    W.init((long long)rows * nqt, gridDim.x, blockIdx.x, nqt);
    const int nb = a.B * a.H;
    auto geom = [&](int ii, int* b, int* h, int* qt) {
        const int R = W.row(ii);
        *qt = R % nqt;
        const int bh = R / nqt;
        *h = bh % a.H;
        *b = bh / a.H;
    };

    if (threadIdx.x == kLoadWarp * 32) {
        for (int i = 0; i < B_COUNT; ++i)
            mbar_init(&bars[i], (i == B_PFULL || i == B_QTM || i == B_ORD || i == B_SREAD || i == B_SREAD + 1)
                                    ? kSoftmaxThreads
                                    : 1);
        *abort_word = 0;
        item_bad[0] = item_bad[1] = 0;
        fence_mbar_init();
        fence_async_smem();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        int b, h, qt;
        geom(0, &b, &h, &qt);
        mbar_expect_tx(&bars[B_Q], kTileBytes);
        tma_load_3d(sb + Q, &tm_q, &bars[B_Q], h * 128, qt * kTile, b);
        tma_load_3d(sb + Q + kHalf, &tm_q, &bars[B_Q], h * 128 + 64, qt * kTile, b);
        for (int t = 0; t < kKStages && t < W.len(0); ++t) {
            const int kt = W.j0(0) + t;
            mbar_expect_tx(&bars[B_KFULL + t], kTileBytes);
            tma_load_3d(sb + K0 + t * kTileBytes, &tm_k, &bars[B_KFULL + t], h * 128, kt * kTile, b);
            tma_load_3d(sb + K0 + t * kTileBytes + kHalf, &tm_k, &bars[B_KFULL + t], h * 128 + 64, kt * kTile, b);
        }
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS0 = tmem, tO = tmem + 256, tQ = tmem + 384, tP = tmem + 448;
    const int ntiles = W.total();

    if (warp == kLoadVWarp) {
        // ------------------------------------------------ TMA producer: V ring
        if (lane == 0) {
            tma_prefetch_desc(&tm_v);
            int ii = 0, t = 0, b = 0, h = 0, qt = 0;
            geom(0, &b, &h, &qt);
            for (int g = 0; g < ntiles && !a.dbg_skip_v; ++g) {
                const int vs = g % kVStages;
                if (g >= kVStages &&
                    !mbar_wait(&bars[B_VEMPTY + vs], ((g / kVStages) + 1) & 1, abort_word, a.flags, a.wait_ns))
                    break;
                const int kt = W.j0(ii) + t;
                mbar_expect_tx(&bars[B_VFULL + vs], kTileBytes);
                tma_load_3d(sb + V0 + vs * kTileBytes, &tm_v, &bars[B_VFULL + vs], h * 128, kt * kTile, b);
                tma_load_3d(sb + V0 + vs * kTileBytes + kHalf, &tm_v, &bars[B_VFULL + vs], h * 128 + 64, kt * kTile,
                            b);
                if (++t == W.len(ii) && ii + 1 < W.nitems) {
                    t = 0;
                    geom(++ii, &b, &h, &qt);
                }
            }
        }
        __syncwarp();
    } else if (warp == kLoadWarp) {
        // ------------------------------------------------ TMA producer: Q per item, K ring with W
        if (lane == 0) {
            tma_prefetch_desc(&tm_w);
            bool ok = true, primary_done = false;
            bool q_next = false;  // the next item's Q is in flight
            int p = 0;            // position in the K ring's sequence
            auto load_q = [&](int jj) {
                int b, h, qt;
                geom(jj, &b, &h, &qt);
                mbar_expect_tx(&bars[B_Q], kTileBytes);
                tma_load_3d(sb + Q, &tm_q, &bars[B_Q], h * 128, qt * kTile, b);
                tma_load_3d(sb + Q + kHalf, &tm_q, &bars[B_Q], h * 128 + 64, qt * kTile, b);
            };
            for (int ii = 0; ii < W.nitems && ok; ++ii) {
                int b, h, qt;
                geom(ii, &b, &h, &qt);
                const int bh = b * a.H + h;
                const int len = W.len(ii);
                if (ii > 0 && !q_next) {
                    // the Q buffer is free once the previous item's scores have read it
                    // and its rows are in TMEM
                    ok = mbar_wait(&bars[B_QFREE], (ii - 1) & 1, abort_word, a.flags, a.wait_ns) &&
                         mbar_wait(&bars[B_QTM], (ii - 1) & 1, abort_word, a.flags, a.wait_ns);
                    if (!ok) break;
                    load_q(ii);
                }
                q_next = false;
                for (int t = 0; t < len && ok; ++t, ++p) {
                    if (ii == 0 && t < kKStages) continue;  // issued at entry
                    const int ks = p % kKStages;
                    // the next item's Q, as soon as this item no longer needs the buffer
                    if (!q_next && ii + 1 < W.nitems && mbar_try_wait(smem_u32(&bars[B_QFREE]), ii & 1) &&
                        mbar_try_wait(smem_u32(&bars[B_QTM]), ii & 1)) {
                        load_q(ii + 1);
                        q_next = true;
                    }
                    if (!(ok = mbar_wait(&bars[B_KEMPTY + ks], ((p / kKStages) + 1) & 1, abort_word, a.flags,
                                         a.wait_ns)))
                        break;
                    const int kt = W.j0(ii) + t;
                    mbar_expect_tx(&bars[B_KFULL + ks], kTileBytes);
                    tma_load_3d(sb + K0 + ks * kTileBytes, &tm_k, &bars[B_KFULL + ks], h * 128, kt * kTile, b);
                    tma_load_3d(sb + K0 + ks * kTileBytes + kHalf, &tm_k, &bars[B_KFULL + ks], h * 128 + 64,
                                kt * kTile, b);
                }
                if (!ok) break;
                if (!W.has_oi(ii)) continue;
                // W_hi, W_lo (row-major, MN-major operands) through the ring; W comes from
                // the prep kernel, which may still run when this grid starts
                if (!primary_done) {
                    pdl_wait_primary();
                    primary_done = true;
                }
                for (int w = 0; w < 2 && ok; ++w, ++p) {
                    const int ks = p % kKStages;
                    if (p >= kKStages &&
                        !(ok = mbar_wait(&bars[B_KEMPTY + ks], ((p / kKStages) + 1) & 1, abort_word, a.flags,
                                         a.wait_ns)))
                        break;
                    mbar_expect_tx(&bars[B_KFULL + ks], kTileBytes);
                    tma_load_3d(sb + K0 + ks * kTileBytes, &tm_w, &bars[B_KFULL + ks], 0, 0, w * nb + bh);
                    tma_load_3d(sb + K0 + ks * kTileBytes + kHalf, &tm_w, &bars[B_KFULL + ks], 64, 0, w * nb + bh);
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_KK = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t ID_KMN = idesc_bf16(128, 128, 0, 1);
            // what each S buffer holds: 1 = a tile's scores (its use number of the
            // buffer, and its tile), 2 = an item's O_inter (the item)
            // (scalars, not arrays indexed by a run-time buffer number, which would
            // live in local memory)
            int kind0 = 0, kind1 = 0, idx0 = 0, idx1 = 0, tile0 = -1, tile1 = -1;
            int uses0 = 0, uses1 = 0;
            int items_pv = 0;  // items whose last P V product is issued
            int items_oi = 0;  // items whose O_inter product is issued
            int sg = 0, s_ii = 0, s_t = 0;
            bool ok = true;
            auto wait_free = [&](int buf) -> bool {
                const int kind = buf ? kind1 : kind0, idx = buf ? idx1 : idx0;
                if (kind == 1) return mbar_wait(&bars[B_SREAD + buf], idx & 1, abort_word, a.flags, a.wait_ns);
                if (kind == 2) return mbar_wait(&bars[B_ORD], idx & 1, abort_word, a.flags, a.wait_ns);
                return true;
            };
            // the scores of tile sg may be issued while P V of tile g is next: at
            // most two tiles ahead, into a buffer whose scores the softmax has read
            // by the time it works on tile g, or whose O_inter belongs to an item
            // whose products are all issued (its epilogue then reads it)
            // (and never into an item's O_inter buffer before that product: a later
            // item's scores wait until every earlier item's O_inter is issued)
            auto can_issue = [&](int g) -> bool {
                if (sg >= ntiles || sg > g + 2 || s_ii > items_oi) return false;
                const int buf = (sg + s_ii) & 1;
                const int kind = buf ? kind1 : kind0, idx = buf ? idx1 : idx0, tile = buf ? tile1 : tile0;
                if (kind == 1 && tile > g) return false;
                if (kind == 2 && idx >= items_pv) return false;
                return true;
            };
            auto issue_s = [&]() -> bool {
                const int buf = (sg + s_ii) & 1;
                if (!wait_free(buf)) return false;
                const int p = W.kbase(s_ii) + s_t;
                const int ks = p % kKStages;
                if (!mbar_wait(&bars[B_KFULL + ks], (p / kKStages) & 1, abort_word, a.flags, a.wait_ns)) return false;
                const bool from_smem = s_t < 2;
                if (!mbar_wait(&bars[from_smem ? B_Q : B_QTM], s_ii & 1, abort_word, a.flags, a.wait_ns))
                    return false;
                tc_fence_after();
                if (from_smem) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tS0 + buf * 128, kmajor_desc(sb + Q, kk), kmajor_desc(sb + K0 + ks * kTileBytes, kk),
                                 ID_KK, kk > 0);
                } else {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tS0 + buf * 128, tQ + kk * 8, kmajor_desc(sb + K0 + ks * kTileBytes, kk), ID_KK,
                                    kk > 0);
                }
                mma_commit(&bars[B_SFULL + buf]);
                mma_commit(&bars[B_KEMPTY + ks]);
                const int len = W.len(s_ii);
                if (s_t == (len < 2 ? len - 1 : 1)) mma_commit(&bars[B_QFREE]);  // last read of Q in shared memory
                if (buf) {
                    kind1 = 1;
                    idx1 = uses1++;
                    tile1 = sg;
                } else {
                    kind0 = 1;
                    idx0 = uses0++;
                    tile0 = sg;
                }
                ++sg;
                if (++s_t == len) {
                    s_t = 0;
                    ++s_ii;
                }
                return true;
            };
            int ii = 0, t = 0;
            for (int g = 0; g < ntiles && ok; ++g) {
                const int len = W.len(ii);
                // at an item's last tile its P V product goes first: the next item's
                // scores (their Q and K may still be in flight) wait one iteration
                // (the item's own scores are always issued)
                const bool ahead = t != len - 1;
                while (ok && (ahead || s_ii <= ii) && can_issue(g)) ok = issue_s();
                if (!ok) break;
                if (t == (len >= 2 ? len - 2 : 0) && !W.has_oi(ii)) {
                    items_oi = ii + 1;  // no O_inter: later items' scores may go ahead
                    while (ok && (ahead || s_ii <= ii) && can_issue(g)) ok = issue_s();
                    if (!ok) break;
                } else if (t == (len >= 2 ? len - 2 : 0)) {
                    // O_inter = Q W_hi + Q W_lo into the S buffer the item's last tile does not use
                    const int boi = (W.gbase(ii) + len + ii) & 1;
                    const int p = W.kbase(ii) + len;  // W_hi, then W_lo
                    const int ks_hi = p % kKStages, ks_lo = (p + 1) % kKStages;
                    if (!(ok = wait_free(boi))) break;
                    if (!(ok = mbar_wait(&bars[B_QTM], ii & 1, abort_word, a.flags, a.wait_ns))) break;
                    if (!(ok = mbar_wait(&bars[B_KFULL + ks_hi], (p / kKStages) & 1, abort_word, a.flags, a.wait_ns)))
                        break;
                    if (!(ok = mbar_wait(&bars[B_KFULL + ks_lo], ((p + 1) / kKStages) & 1, abort_word, a.flags,
                                         a.wait_ns)))
                        break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tS0 + boi * 128, tQ + kk * 8, mnmajor_desc(sb + K0 + ks_hi * kTileBytes, kk),
                                    ID_KMN, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tS0 + boi * 128, tQ + kk * 8, mnmajor_desc(sb + K0 + ks_lo * kTileBytes, kk),
                                    ID_KMN, 1);
                    mma_commit(&bars[B_OIDONE]);
                    mma_commit(&bars[B_KEMPTY + ks_hi]);
                    mma_commit(&bars[B_KEMPTY + ks_lo]);
                    if (boi) {
                        kind1 = 2;
                        idx1 = ii;
                    } else {
                        kind0 = 2;
                        idx0 = ii;
                    }
                    items_oi = ii + 1;
                    while (ok && (ahead || s_ii <= ii) && can_issue(g)) ok = issue_s();
                    if (!ok) break;
                }
                // O is free for the item's first product once the previous epilogue read it
                if (t == 0 && ii > 0 && !(ok = mbar_wait(&bars[B_ORD], (ii - 1) & 1, abort_word, a.flags, a.wait_ns)))
                    break;
                const int vs = g % kVStages;
                if (!(ok = mbar_wait(&bars[B_PFULL], g & 1, abort_word, a.flags, a.wait_ns))) break;
                if (!(ok = mbar_wait(&bars[B_VFULL + vs], (g / kVStages) & 1, abort_word, a.flags, a.wait_ns))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tO, tP + kk * 8, mnmajor_desc(sb + V0 + vs * kTileBytes, kk), ID_KMN, (t > 0 || kk > 0));
                mma_commit(&bars[B_PVDONE]);
                mma_commit(&bars[B_VEMPTY + vs]);
                if (++t == len) {
                    t = 0;
                    items_pv = ++ii;
                }
            }
            // drain: every MMA issued so far completes before TMEM is released
            mma_commit(&bars[B_DRAIN]);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&bars[B_DRAIN]), 0) && globaltimer_ns() - t0 < a.wait_ns) {
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax + epilogue
        // The per-tile work is that of tc_attention.cuh (a row per pair of warps,
        // a running offset that moves only when a half row's partial sum leaves
        // [0, 2^63), codes exchanged per tile at the pair barrier); the tile's S
        // buffer and exchange slot are (tile + item) & 1 over the CTA's sequence.
        const int gq = warp & 3, hf = warp >> 2;
        const int r = gq * 32 + lane;
        const int pair_bar = 1 + gq;
        const uint32_t lrow = (uint32_t)(gq * 32) << 16;
        const uint32_t cs = hf * 64;
        float* xch = (float*)(smem + XCH);
        uint8_t* xfl = smem + XFL;
        const int mine = hf * 128 + r, theirs = (hf ^ 1) * 128 + r;
        const float scale = a.sm_scale_log2;
        int uses0 = 0, uses1 = 0;  // tiles read from S buffer 0 / 1 so far
        int tail_old = 0;          // thread 0: the tail's ticket (taken without waiting for it)
        bool tail_pub = false;
        bool ok = true;
        int gt = 0;  // this item's first tile in the CTA's sequence
        float x[64];
        for (int ii = 0; ii < W.nitems; ++ii) {
            int b, h, qt;
            geom(ii, &b, &h, &qt);
            const int bh = b * a.H + h;
            const int len = W.len(ii), j0 = W.j0(ii);
            const bool partial = j0 > 0 || W.j1(ii) < nqt;
            float m = 0.f, l = 0.f;
            // Q half-row into TMEM (the previous epilogue waited for every product
            // of the previous item, so nothing reads TMEM Q any more)
            ok = ok && __all_sync(0xffffffffu, mbar_wait(&bars[B_Q], ii & 1, abort_word, a.flags, a.wait_ns));
            if (ok) {
                uint32_t qv[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4*>(smem + Q + hf * kHalf + sw128_offset(r, c));
                    qv[4 * c] = v.x;
                    qv[4 * c + 1] = v.y;
                    qv[4 * c + 2] = v.z;
                    qv[4 * c + 3] = v.w;
                }
                tmem_st32u(tQ + lrow + hf * 32, qv);
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(&bars[B_QTM]);
            {
                const int s0 = (gt + ii) & 1;
                ok = ok && __all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL + s0], (s0 ? uses1 : uses0) & 1,
                                                             abort_word, a.flags, a.wait_ns));
                if (ok) {
                    tc_fence_after();
                    tmem_ld32(tS0 + s0 * 128 + lrow + cs, x);
                    tmem_ld32(tS0 + s0 * 128 + lrow + cs + 32, x + 32);
                }
            }
            for (int t = 0; t < len; ++t) {
                const int g = gt + t;
                const int s = (g + ii) & 1;
                if (s) ++uses1;
                else ++uses0;
                const bool w_ok = ok;
                uint32_t pk[32];
                float lt = 0.f;
                if (w_ok) {
                    tmem_ld_wait();
                    tc_fence_before();
                    mbar_arrive(&bars[B_SREAD + s]);
                    const int valid = T - (j0 + t) * kTile - (int)cs;
                    if (valid < 64) {
#pragma unroll
                        for (int c = 0; c < 64; ++c)
                            if (c >= valid) x[c] = -INFINITY;
                    }
                }
                if (t == 0) {
                    const float hm = w_ok ? row_max<64>(x) : -INFINITY;
                    xch[s * 256 + mine] = hm;
                    named_bar_sync(pair_bar, 64);
                    m = fmaxf(hm, xch[s * 256 + theirs]) * scale;
                }
                bool redo_h = false;
                if (w_ok) {
                    lt = exp_scores<64>(x, scale, -m, pk);
                    redo_h = !(lt < 9.2233720e18f);
                }
                xfl[s * 256 + mine] = w_ok ? (redo_h ? 2 : 1) : 0;
                named_bar_sync(pair_bar, 64);
                const uint8_t pc = xfl[s * 256 + theirs];
                ok = __all_sync(0xffffffffu, w_ok && pc != 0);
                const bool redo = ok && (redo_h || pc == 2);
                const bool any_redo = __any_sync(0xffffffffu, redo);
                float f = 1.0f;
                if (any_redo) {
                    const float hm = redo ? row_max<64>(x) * scale : -INFINITY;
                    xch[s * 256 + mine] = hm;
                    named_bar_sync(pair_bar, 64);
                    if (redo) {
                        const float mn = fmaxf(m, fmaxf(hm, xch[s * 256 + theirs]));
                        f = ex2(m - mn);
                        m = mn;
                    }
                    lt = exp_scores<64>(x, scale, -m, pk);
                }
                if (!ok) continue;
                l = fmaf(l, f, lt);
                if (t > 0) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PVDONE], (g - 1) & 1, abort_word, a.flags, a.wait_ns));
                    if (!ok) continue;
                    tc_fence_after();
                }
                if (any_redo && t > 0) {
#pragma unroll 1
                    for (int c = 0; c < 64; c += 32) {
                        float o[32];
                        tmem_ld32(tO + lrow + cs + c, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 32; ++q) o[q] *= f;
                        tmem_st32(tO + lrow + cs + c, o);
                    }
                }
                tmem_st32u(tP + lrow + hf * 32, pk);
                if (t + 1 < len) {
                    const int s1 = s ^ 1;
                    ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL + s1], (s1 ? uses1 : uses0) & 1,
                                                           abort_word, a.flags, a.wait_ns));
                    if (ok) {
                        tc_fence_after();
                        tmem_ld32(tS0 + s1 * 128 + lrow + cs, x);
                        tmem_ld32(tS0 + s1 * 128 + lrow + cs + 32, x + 32);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                if (ok) mbar_arrive(&bars[B_PFULL]);
            }
            gt += len;
            // ---------------------------------------------------- epilogue of the item
            const int p = (gt + ii) & 1;  // exchange slot after the item's last tile
            const bool has_oi = W.has_oi(ii);
            const uint32_t tOI = tS0 + p * 128;
            const int par = ii & 1;
            const int slot = (ii == 0 && j0 > 0) ? (int)blockIdx.x : (int)blockIdx.x + 1;  // the split's boundary
            const bool tail = ii == 0 && j0 > 0;
            int* cnt = a.sk_cnt + slot;
            // a head's look at the split row's ticket (read early: its latency overlaps the
            // waits; a schedule test may skip it)
            int peek = 0;
            if (partial && !tail && threadIdx.x == 0 && a.dbg_sk_mode != 2) peek = ld_acquire_gpu(cnt);
            // the CTA's last item: the K and V rings and the Q buffer are free once its
            // last P V product is done; the output goes through the Q buffer and two TMA
            // stores, and a head whose tail has finished copies the tail's record into
            // the rings while the ticket is taken
            const bool last = ii == W.nitems - 1;
            const bool pull = last && partial && !tail;
            if (ok) tmem_ld_wait();
            bool e_ok = ok && mbar_wait(&bars[B_PVDONE], (gt - 1) & 1, abort_word, a.flags, a.wait_ns);
            e_ok = __all_sync(0xffffffffu,
                              e_ok && (!has_oi || mbar_wait(&bars[B_OIDONE], (ii - (W.j0_first > 0 ? 1 : 0)) & 1,
                                                            abort_word, a.flags, a.wait_ns)));
            bool pulled = false;  // thread 0: the tail's record is on its way into shared memory
            if (pull && threadIdx.x == 0 && peek != 0 && e_ok) {
                fence_proxy_async_global();
                mbar_expect_tx(&bars[B_REC], kTailBytes);
                bulk_load(sb + K0, a.sk_part + (size_t)slot * kSlotFloats + kHeadFloats, kTailBytes, &bars[B_REC]);
                pulled = true;
            }
            xch[p * 256 + mine] = l;
            xfl[p * 256 + mine] = e_ok ? 1 : 0;
            named_bar_sync(pair_bar, 64);
            const bool both = __all_sync(0xffffffffu, e_ok && xfl[p * 256 + theirs] != 0);
            const float lrow_sum = l + xch[p * 256 + theirs];
            if (!both && lane == 0) item_bad[par] = 1;
            if (partial && threadIdx.x == 0) ticket[par * 2] = peek;
            named_bar_sync(5, kSoftmaxThreads);
            const bool bad = item_bad[par] != 0;
            if (threadIdx.x == 0) item_bad[par ^ 1] = 0;  // for the next item (no thread reads it before then)
            const int t_row = qt * kTile + r;
            const float gain = a.mix ? a.mix[bh * 2] : 1.0f;
            __nv_bfloat16* orow =
                reinterpret_cast<__nv_bfloat16*>(a.out) + (((size_t)b * T + t_row) * a.H + h) * 128 + cs;
            tc_fence_after();
            // 16 bytes (8 output columns, unit u of this half row): staged in the Q buffer
            // (128B-swizzled, as the output tensor map's box) for the last item, else
            // stored directly (rows past T skipped)
            auto put = [&](int u, const uint4& w) {
                if (last)
                    *reinterpret_cast<uint4*>(smem + Q + hf * kHalf + sw128_offset(r, u)) = w;
                else if (t_row < T)
                    reinterpret_cast<uint4*>(orow)[u] = w;
            };
            // out = O / l + O_inter, 16 columns at a time, O_inter from TMEM
            auto store_out = [&](float lsum) {
                const float inv_out = (1.0f / lsum) * gain;  // as the one-CTA-per-tile kernel rounds it
#pragma unroll 1
                for (int c0 = 0; c0 < 64; c0 += 16) {
                    float o[16], e[16];
                    tmem_ld16(tO + lrow + cs + c0, o);
                    tmem_ld16(tOI + lrow + cs + c0, e);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint4 w;
                        w.x = pack_bf16(o[8 * q + 0] * inv_out + e[8 * q + 0], o[8 * q + 1] * inv_out + e[8 * q + 1]);
                        w.y = pack_bf16(o[8 * q + 2] * inv_out + e[8 * q + 2], o[8 * q + 3] * inv_out + e[8 * q + 3]);
                        w.z = pack_bf16(o[8 * q + 4] * inv_out + e[8 * q + 4], o[8 * q + 5] * inv_out + e[8 * q + 5]);
                        w.w = pack_bf16(o[8 * q + 6] * inv_out + e[8 * q + 6], o[8 * q + 7] * inv_out + e[8 * q + 7]);
                        put(c0 / 8 + q, w);
                    }
                }
            };
            // a head's merge: out = (O fh + O_tail ft) / lsum + O_inter, 32 columns at a
            // time with the tail's O (record matrix, in shared memory if it was copied
            // there) loaded up front for each 32; the same order of operations as a
            // tail's deferred merge
            auto store_merged = [&](float fh, float ft, float lsum, const float* oth, bool in_smem) {
                const float inv_out = (1.0f / lsum) * gain;
#pragma unroll 1
                for (int c1 = 0; c1 < 64; c1 += 32) {
                    float4 u[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int f = ((cs + c1) / 4 + q) * 128 + r;
                        u[q] = in_smem ? reinterpret_cast<const float4*>(smem + K0)[f]
                                       : __ldcg(reinterpret_cast<const float4*>(oth) + f);
                    }
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int c0 = c1 + 16 * h2;
                        float o[16], e[16];
                        tmem_ld16(tO + lrow + cs + c0, o);
                        tmem_ld16(tOI + lrow + cs + c0, e);
                        tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 v = u[4 * h2 + q];
                            o[4 * q] = fmaf(o[4 * q], fh, v.x * ft);
                            o[4 * q + 1] = fmaf(o[4 * q + 1], fh, v.y * ft);
                            o[4 * q + 2] = fmaf(o[4 * q + 2], fh, v.z * ft);
                            o[4 * q + 3] = fmaf(o[4 * q + 3], fh, v.w * ft);
                        }
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            uint4 w;
                            w.x = pack_bf16(o[8 * q + 0] * inv_out + e[8 * q + 0], o[8 * q + 1] * inv_out + e[8 * q + 1]);
                            w.y = pack_bf16(o[8 * q + 2] * inv_out + e[8 * q + 2], o[8 * q + 3] * inv_out + e[8 * q + 3]);
                            w.z = pack_bf16(o[8 * q + 4] * inv_out + e[8 * q + 4], o[8 * q + 5] * inv_out + e[8 * q + 5]);
                            w.w = pack_bf16(o[8 * q + 6] * inv_out + e[8 * q + 6], o[8 * q + 7] * inv_out + e[8 * q + 7]);
                            put(c0 / 8 + q, w);
                        }
                    }
                }
            };
            bool wrote = false;  // this item's output tile is computed (uniform over the CTA)
            if (!partial) {
                wrote = !bad;
                if (wrote) store_out(lrow_sum);
            } else {
                // A split row.  The tail (its CTA's first item) always publishes its record
                // and takes its ticket without waiting for it; it looks at the ticket after
                // its CTA's last item and merges there, from the two records, if the head
                // took the first ticket.  The head merges at once if it has seen the tail's
                // ticket; otherwise it publishes (O_inter too), takes its ticket and merges
                // if that ticket is the second.  Writes of a record by every thread are
                // ordered before thread 0's release (the barrier, then its ticket); a
                // merging CTA reads after its thread 0's acquire (the look or the ticket)
                // and the barrier.
                float* rec = a.sk_part + (size_t)slot * kSlotFloats + (tail ? kHeadFloats : 0);
                const float* tl = a.sk_part + (size_t)slot * kSlotFloats + kHeadFloats;
                const bool seen = !tail && ticket[par * 2] != 0;  // a head that saw the tail's ticket
                if (!seen && !bad) {
#pragma unroll 1
                    for (int c0 = 0; c0 < 64; c0 += 16) {
                        float o[16];
                        tmem_ld16(tO + lrow + cs + c0, o);
                        tmem_ld_wait();
                        float4* dst = reinterpret_cast<float4*>(rec) + ((cs + c0) / 4) * 128 + r;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q * 128] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
                        if (!tail) {
                            // the head's O_inter, for a tail that merges
                            tmem_ld16(tOI + lrow + cs + c0, o);
                            tmem_ld_wait();
                            float4* dsti = reinterpret_cast<float4*>(rec + kRecOI) + ((cs + c0) / 4) * 128 + r;
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                dsti[q * 128] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
                        }
                    }
                    if (hf == 0) {
                        rec[kRecM + r] = m;
                        rec[kRecL + r] = lrow_sum;
                    }
                }
                named_bar_sync(5, kSoftmaxThreads);
                if (threadIdx.x == 0) {
                    int old = seen ? 1 : 0;
                    if (!seen) {
                        reinterpret_cast<volatile int*>(rec)[kRecOk] = bad ? 0 : 1;
                        if (!tail)
                            old = atomic_add_acq_rel_gpu(cnt, 1);
                        else if (a.dbg_sk_mode != 1)  // (a schedule test may hold it to the CTA's end)
                            tail_old = atomic_add_release_gpu(cnt, 1);
                        tail_pub = tail_pub || tail;
                    }
                    if (old != 0) *cnt = 0;  // this CTA merges: the row's ticket is spent
                    ticket[par * 2 + 1] = old;
                }
                named_bar_sync(5, kSoftmaxThreads);
                if (!tail && ticket[par * 2 + 1] != 0) {
                    // the tail's record is complete: merge (from shared memory if it was
                    // copied there)
                    const bool in_smem = pull && seen && !bad;
                    bool got = true;
                    if (in_smem) got = __all_sync(0xffffffffu, mbar_wait(&bars[B_REC], 0, abort_word, a.flags, a.wait_ns));
                    const float* src = in_smem ? reinterpret_cast<const float*>(smem + K0) : tl;
                    const float mt = in_smem ? src[kRecM + r] : __ldcg(src + kRecM + r);
                    const float lt = in_smem ? src[kRecL + r] : __ldcg(src + kRecL + r);
                    const int ok_t = in_smem ? reinterpret_cast<const int*>(src)[kRecOk]
                                             : __ldcg(reinterpret_cast<const int*>(src) + kRecOk);
                    const float mm = fmaxf(m, mt);
                    const float fh = ex2(m - mm), ft = ex2(mt - mm);
                    wrote = !bad && got && ok_t;
                    if (wrote) store_merged(fh, ft, fmaf(lrow_sum, fh, lt * ft), tl, in_smem);
                }
            }
            if (pulled) mbar_wait(&bars[B_REC], 0, abort_word, a.flags, a.wait_ns);  // no copy left in flight
            if (last) {
                // the staged output tile: two TMA stores (rows past T are clipped by the map)
                fence_async_smem();
                named_bar_sync(5, kSoftmaxThreads);
                if (threadIdx.x == 0 && wrote) {
                    tma_store_3d(&tm_o, sb + Q, h * 128, qt * kTile, b);
                    tma_store_3d(&tm_o, sb + Q + kHalf, h * 128 + 64, qt * kTile, b);
                    bulk_commit_group();
                    bulk_wait_read_all();
                }
            }
            // O and O_inter are read: the next item may overwrite them
            tc_fence_before();
            mbar_arrive(&bars[B_ORD]);
        }
        // A tail whose ticket came second (the head finished first and published):
        // its row's output from the two records, in the same order of operations as a
        // merge by either segment.
        if (W.j0_first > 0) {
            volatile int* deferred = (volatile int*)(tmem_slot + 8);
            if (threadIdx.x == 0) {
                // (a schedule test holds the tail's ticket to here, after the head's)
                if (tail_pub && a.dbg_sk_mode == 1) tail_old = atomic_add_acq_rel_gpu(a.sk_cnt + blockIdx.x, 1);
                int v = tail_pub ? tail_old : 0;
                if (v != 0) {
                    fence_acq_rel_gpu();
                    a.sk_cnt[blockIdx.x] = 0;
                }
                *deferred = v;
            }
            named_bar_sync(5, kSoftmaxThreads);
            if (*deferred != 0) {
                int b, h, qt;
                geom(0, &b, &h, &qt);
                const int bh = b * a.H + h;
                const float* head = a.sk_part + (size_t)blockIdx.x * kSlotFloats;
                const float* tl = head + kHeadFloats;
                const float mh = __ldcg(head + kRecM + r), lh = __ldcg(head + kRecL + r);
                const float mt = __ldcg(tl + kRecM + r), lt = __ldcg(tl + kRecL + r);
                const int ok2 = __ldcg(reinterpret_cast<const int*>(head) + kRecOk) &
                                __ldcg(reinterpret_cast<const int*>(tl) + kRecOk);
                const float mm = fmaxf(mh, mt);
                const float fh = ex2(mh - mm), ft = ex2(mt - mm);
                const float inv_out = (1.0f / fmaf(lh, fh, lt * ft)) * (a.mix ? a.mix[bh * 2] : 1.0f);
                const int t_row = qt * kTile + r;
                uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) +
                                                       (((size_t)b * T + t_row) * a.H + h) * 128 + cs);
                if (ok2 && t_row < T) {
#pragma unroll 1
                    for (int u = 0; u < 8; ++u) {  // 8 output columns at a time
                        float y[8], e[8];
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int f = ((int)cs / 4 + 2 * u + q) * 128 + r;
                            const float4 oh = __ldcg(reinterpret_cast<const float4*>(head) + f);
                            const float4 ot = __ldcg(reinterpret_cast<const float4*>(tl) + f);
                            const float4 oi = __ldcg(reinterpret_cast<const float4*>(head + kRecOI) + f);
                            y[4 * q] = fmaf(oh.x, fh, ot.x * ft);
                            y[4 * q + 1] = fmaf(oh.y, fh, ot.y * ft);
                            y[4 * q + 2] = fmaf(oh.z, fh, ot.z * ft);
                            y[4 * q + 3] = fmaf(oh.w, fh, ot.w * ft);
                            e[4 * q] = oi.x;
                            e[4 * q + 1] = oi.y;
                            e[4 * q + 2] = oi.z;
                            e[4 * q + 3] = oi.w;
                        }
                        uint4 w;
                        w.x = pack_bf16(y[0] * inv_out + e[0], y[1] * inv_out + e[1]);
                        w.y = pack_bf16(y[2] * inv_out + e[2], y[3] * inv_out + e[3]);
                        w.z = pack_bf16(y[4] * inv_out + e[4], y[5] * inv_out + e[5]);
                        w.w = pack_bf16(y[6] * inv_out + e[6], y[7] * inv_out + e[7]);
                        orow[u] = w;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace tc
}  // namespace hyb
