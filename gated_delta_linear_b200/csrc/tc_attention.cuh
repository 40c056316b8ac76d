// tc_attention.cuh -- intra-frame softmax attention with the inter-frame read
// fused into its epilogue, for bf16 I/O and d = 128 on sm_100a.
//
// Source: "Technical summary: Attend Locally, Remember Linearly (ARL2)",
// gist.science/ar/paper/2605.16579, §2.1: the intra-frame branch is the
// original bidirectional softmax attention over the tokens of the frame; the
// inter-frame branch reads O_inter = Q' S_{N-1} = Q (phi_q^T S_{N-1}) (§2.2:
// every token reads the same pre-update state).  The layer output is
// O_intra + O_inter (the pages leave the combination open; this library sums).
//
// attention_kernel: one CTA per (128-query tile, head, batch), 11 warps (the
// kMulti variant: per run of consecutive query tiles of a head, taken one after
// another, each as below).
// Warp 8 streams Q and the K ring, warp 10 the V ring, with TMA into
// 128B-swizzled shared memory; warp 9 issues the tcgen05 MMAs; warps 0-7 run
// the online softmax, a query row per pair of threads (warps w and w+4, 64
// scores each in registers).  Near the end of the key loop the Q tile is
// multiplied by W = phi_q^T S_{N-1} (a two-term bf16 split W_hi + W_lo, row
// major: an MN-major B operand), so the inter-frame read lands in TMEM next to
// the softmax accumulator and the epilogue writes out = O_intra + O_inter once.
//   TMEM columns: [0,128) S buffer 0, [128,256) S buffer 1, [256,384) O,
//                 [384,448) P buffer 0, [448,512) P buffer 1 (bf16, two per
//                 32-bit column: the A operand of O += P V).  S = Q K^T takes
//                 both operands from shared memory.  As soon as the softmax has
//                 S_j in registers the MMA warp issues S_{j+2} into its buffer,
//                 so scores run a tile ahead of the softmax, and the softmax
//                 loads S_{j+1} while it hands P_j over.  P_j goes to buffer
//                 j & 1, so the softmax never waits for P_{j-1} V_{j-1}: the
//                 value product of one tile runs while the next tile's P is
//                 written, and the tensor pipe is not idle for the round trip
//                 from one value product's completion to the next P.
//   Softmax: exponents against a running offset (the first tile's row max),
//                 moved only when a tile's partial sum over a half row leaves
//                 [0, 2^63); all exponentials on the MUFU pipe.
//   Shared memory: Q 32 KB | K 3 x 32 KB | V 3 x 32 KB.  Near the end W_hi
//                 and W_lo take the K stages of key tiles n-3 and n-2 (unused
//                 stages when n < 3) and O_inter = Q W_hi + Q W_lo goes to the
//                 S buffer the last tile does not use while the softmax works
//                 on the last two tiles; the bf16 output tile is assembled in
//                 the Q buffer and written with two TMA stores.
//   Token-level access (a.oi_ext): no W product; the epilogue adds the fp32
//                 read the token-level kernels computed.
//   Every CTA signals at entry that the next kernel (the delta update, which
//   reads none of this kernel's outputs) may start on idle SMs.
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tc_kernels.cuh"

namespace hyb {
namespace tc {

using namespace sm100;

namespace attn {
constexpr int kKStages = 3;                    // K ring depth
constexpr int kVStages = 3;                    // V ring depth
constexpr uint32_t Q = 0;
constexpr uint32_t K0 = Q + kTileBytes;
constexpr uint32_t V0 = K0 + kKStages * kTileBytes;
constexpr uint32_t BAR = V0 + kVStages * kTileBytes;
constexpr uint32_t XCH = BAR + 256;            // softmax pair exchange: [2 parity][2 halves][128 rows] floats
constexpr uint32_t XFL = XCH + 2048;           // and codes [2][2][128] bytes
constexpr uint32_t SMEM = XFL + 512;           // 232,192 B
constexpr int kSoftmaxThreads = 256;           // warps 0-7: rows 32(w&3)..+31, column half w>>2
constexpr int kLoadWarp = 8, kMmaWarp = 9, kLoadVWarp = 10;
constexpr int kThreads = 352;
enum { B_Q = 0, B_W = 1, B_OIDONE = 2, B_KFULL = 3, B_KEMPTY = 6, B_VFULL = 9, B_VEMPTY = 12, B_SFULL = 15,
       B_SREAD = 17, B_PFULL = 19, B_PVDONE = 21, B_OFREE = 23, B_QFREE = 24, B_DRAIN = 25, B_COUNT = 26 };
// per P buffer j & 1: B_PFULL + (j & 1) (P_j written) and B_PVDONE + (j & 1)
// (P_j V_j done).  A softmax warp may run a tile ahead of another, so P_{j+1}
// must not arrive on P_j's barrier; it cannot run two ahead (P_{j+2} waits for
// P_j V_j, which waits for every warp's P_j).
static_assert(B_COUNT * 8 + 8 <= 256, "barrier block");
}  // namespace attn

// p = 2^(x * scale + neg_m) for N scores, as N/2 bf16 pairs (round to
// nearest) in pk; returns the sum of p in fp32 (the exponentials on the MUFU
// pipe, the pair conversion one instruction per two values).
template <int N>
__device__ __forceinline__ float exp_scores(const float* x, float scale, float neg_m, uint32_t* pk) {
    float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < N / 2; ++k) {
        const float e0 = ex2(fmaf(x[2 * k], scale, neg_m));
        const float e1 = ex2(fmaf(x[2 * k + 1], scale, neg_m));
        l4[(2 * k) & 3] += e0;
        l4[(2 * k + 1) & 3] += e1;
        pk[k] = pack_bf16(e0, e1);
    }
    return (l4[0] + l4[1]) + (l4[2] + l4[3]);
}

// The same with the row's sum of p (y - m) in *A (y = x * scale), for the
// attention entropy; masked scores (-inf) give p = 0 and add nothing.
template <int N>
__device__ __forceinline__ float exp_scores_ent(const float* x, float scale, float neg_m, uint32_t* pk, float* A) {
    float l4[4] = {0.f, 0.f, 0.f, 0.f}, a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < N / 2; ++k) {
        const float t0 = fmaxf(fmaf(x[2 * k], scale, neg_m), -1e30f);
        const float t1 = fmaxf(fmaf(x[2 * k + 1], scale, neg_m), -1e30f);
        const float e0 = ex2(t0), e1 = ex2(t1);
        l4[(2 * k) & 3] += e0;
        l4[(2 * k + 1) & 3] += e1;
        a4[(2 * k) & 3] = fmaf(e0, t0, a4[(2 * k) & 3]);
        a4[(2 * k + 1) & 3] = fmaf(e1, t1, a4[(2 * k + 1) & 3]);
        pk[k] = pack_bf16(e0, e1);
    }
    *A = (a4[0] + a4[1]) + (a4[2] + a4[3]);
    return (l4[0] + l4[1]) + (l4[2] + l4[3]);
}

// kEnt: the warm-up pass of Token Radius Attention, which also writes each
// query's attention entropy (a.ent_out).  A key-block list (a.kv_list) makes
// the key loop walk only the listed blocks (block-sparse intra-frame attention).
// kMulti: a CTA takes a.q_per_cta consecutive query tiles, one after another
// (without it the tile loops below run once, and the compiler drops them).
template <bool kEnt, bool kMulti = false>
__global__ void __launch_bounds__(attn::kThreads, 1)
    attention_kernel(const __grid_constant__ LayerArgs a, const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_o) {
    using namespace attn;
    extern __shared__ __align__(1024) uint8_t smem[];
    // 128B-swizzled tiles need a 1024-byte aligned base (the dynamic window starts
    // after the 1 KB reserved block); report and leave if it is not
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicOr(a.flags, FLAG_INTERNAL);
        return;
    }
    // the delta update of this pass does not read anything this kernel writes:
    // it may start on SMs this grid leaves idle
    pdl_launch_dependents();
    const uint32_t sb = smem_u32(smem);
    uint64_t* bars = (uint64_t*)(smem + BAR);
    uint32_t* tmem_slot = (uint32_t*)(bars + B_COUNT);
    volatile int* abort_word = (volatile int*)(tmem_slot + 1);
    volatile int* epi_bad = (volatile int*)(tmem_slot + 2);  // a softmax warp missed its epilogue

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the query tiles of this CTA: nt consecutive tiles from its grid position
    // (a.q_per_cta of them, fewer at the end of a head), or the one row that
    // the schedule of a block-sparse pass gives it
    const int qpc = kMulti && a.q_per_cta > 1 ? a.q_per_cta : 1;
    const int n_qt = (a.T + kTile - 1) / kTile;
    int qt_ = blockIdx.x * qpc, h = blockIdx.y, b = blockIdx.z;
    // (before a mask is built the schedule and the lengths are zero: grid order)
    if (a.kv_order) {
        const int row = a.kv_order[blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z)];
        if (a.kv_count[row] > 0) {
            qt_ = row % n_qt;
            h = (row / n_qt) % a.H;
            b = row / (n_qt * a.H);
        }
    }
    const int nt = min(qpc, n_qt - qt_);
    const int T = a.T;
    auto q0_of = [&](int t) { return (qt_ + t) * kTile; };  // first query row of the CTA's tile t
    const int q0 = q0_of(0);
    const int bh_ = b * a.H + h;
    const size_t kvrow = ((size_t)bh_ * n_qt + qt_);
    // key tiles: every tile of the frame, or the listed ones (block-sparse)
    // (a listed count of 0 means no mask has been built: every tile)
    const int kvc = a.kv_count ? a.kv_count[kvrow] : 0;
    const int n = kvc > 0 ? kvc : (a.T_kv + kTile - 1) / kTile;
    const int* kvl = kvc > 0 ? a.kv_list + kvrow * a.kv_stride : nullptr;
    auto ktile = [&](int j) { return kvl ? kvl[j] : j; };  // frame tile of the j-th key tile walked
    const bool inter = a.inter != 0;             // add O_inter = Q W (hybrid layer)
    const int bh = bh_;
    // Key tile j of the CTA's query tile t is walked as step g = t n + j; every
    // ring stage, TMEM buffer and barrier phase follows g.  K stages that receive
    // W_hi / W_lo at the end of tile t (free once the scores of its key tiles
    // n-3 / n-2 are computed; stages no tile uses when n is small, which only a
    // single-tile CTA meets)
    auto wst_hi_of = [&](int base) { return n >= 3 ? (base + n - 3) % kKStages : 2; };
    auto wst_lo_of = [&](int base) { return n >= 2 ? (base + n - 2) % kKStages : 1; };

    if (threadIdx.x == kLoadWarp * 32) {
        // the producer initialises the barriers and starts the first loads
        // before the block synchronises (the loads land on its own barriers)
        for (int i = 0; i < B_COUNT; ++i)
            mbar_init(&bars[i], (i == B_PFULL || i == B_PFULL + 1 || i == B_SREAD || i == B_SREAD + 1 || i == B_OFREE)
                                    ? kSoftmaxThreads
                                    : 1);
        *abort_word = 0;
        *epi_bad = 0;
        fence_mbar_init();
        fence_async_smem();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        const int xh = h * 128;
        mbar_expect_tx(&bars[B_Q], kTileBytes);
        tma_load_3d(sb + Q, &tm_q, &bars[B_Q], xh, q0, b);
        tma_load_3d(sb + Q + kHalf, &tm_q, &bars[B_Q], xh + 64, q0, b);
        for (int j = 0; j < kKStages && j < n; ++j) {
            mbar_expect_tx(&bars[B_KFULL + j], kTileBytes);
            tma_load_3d(sb + K0 + j * kTileBytes, &tm_k, &bars[B_KFULL + j], xh, ktile(j) * kTile, b);
            tma_load_3d(sb + K0 + j * kTileBytes + kHalf, &tm_k, &bars[B_KFULL + j], xh + 64, ktile(j) * kTile, b);
        }
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // S buffers 0 / 1, O, and P buffers 0 / 1 as bf16 pairs (P_j in buffer j & 1:
    // the A operand of O += P_j V_j)
    const uint32_t tS0 = tmem, tO = tmem + 256, tP = tmem + 384;
    // O_inter of tile t: the S buffer its last key tile does not use
    auto tOI_of = [&](int base) { return tS0 + ((base + n) & 1) * 128; };
    // (producers) the last step whose V / K tile was issued (the first K tiles at
    // entry), the last query tile whose Q and W were issued: after a wait gave
    // up, these loads may still be landing when the block ends
    int vg_last = -1, kg_last = (n < kKStages ? n : kKStages) - 1, q_last = 0, w_last = -1;

    if (warp == kLoadVWarp) {
        // ------------------------------------------------ TMA producer: V ring
        if (lane == 0) {
            tma_prefetch_desc(&tm_v);
            const int xh = h * 128;
            // (a fault test may switch this producer off: the MMA issuer's wait for V
            // then expires, and the kernel reports a timeout and unwinds)
            for (int g = 0; g < nt * n && !a.dbg_skip_v; ++g) {
                const int vs = g % kVStages, kt = ktile(g % n);
                if (g >= kVStages &&
                    !mbar_wait(&bars[B_VEMPTY + vs], ((g / kVStages) + 1) & 1, abort_word, a.flags, a.wait_ns))
                    break;
                mbar_expect_tx(&bars[B_VFULL + vs], kTileBytes);
                tma_load_3d(sb + V0 + vs * kTileBytes, &tm_v, &bars[B_VFULL + vs], xh, kt * kTile, b);
                tma_load_3d(sb + V0 + vs * kTileBytes + kHalf, &tm_v, &bars[B_VFULL + vs], xh + 64, kt * kTile, b);
                vg_last = g;
            }

        }
        __syncwarp();
    } else if (warp == kLoadWarp) {
        // ------------------------------------------------ TMA producer: Q, K ring, W
        // (its own warp, so K tiles run ahead of the V ring's waits)
        if (lane == 0) {
            tma_prefetch_desc(&tm_w);
            const int xh = h * 128;
            const int nbh = a.B * a.H;
            bool ok = true;
            for (int t = 0; t < nt && ok; ++t) {
                const int base = t * n;
                if (t > 0) {
                    // the next query tile goes into the Q buffer once the previous
                    // tile's output has been read out of it, and its first key tiles
                    // into the K stages that held the previous tile's W once the
                    // inter-frame product has read them
                    if (!(ok = mbar_wait(&bars[B_QFREE], (t - 1) & 1, abort_word, a.flags, a.wait_ns))) break;
                    mbar_expect_tx(&bars[B_Q], kTileBytes);
                    tma_load_3d(sb + Q, &tm_q, &bars[B_Q], xh, q0_of(t), b);
                    tma_load_3d(sb + Q + kHalf, &tm_q, &bars[B_Q], xh + 64, q0_of(t), b);
                    q_last = t;
                    if (inter && !(ok = mbar_wait(&bars[B_OIDONE], (t - 1) & 1, abort_word, a.flags, a.wait_ns)))
                        break;
                }
                // (Q and K_0..K_2 of the first tile were issued at entry)
                for (int j = t == 0 ? kKStages : 0; j < n && ok; ++j) {
                    const int g = base + j, ks = g % kKStages;
                    if (!(ok = mbar_wait(&bars[B_KEMPTY + ks], ((g / kKStages) + 1) & 1, abort_word, a.flags,
                                         a.wait_ns)))
                        break;
                    mbar_expect_tx(&bars[B_KFULL + ks], kTileBytes);
                    tma_load_3d(sb + K0 + ks * kTileBytes, &tm_k, &bars[B_KFULL + ks], xh, ktile(j) * kTile, b);
                    tma_load_3d(sb + K0 + ks * kTileBytes + kHalf, &tm_k, &bars[B_KFULL + ks], xh + 64,
                                ktile(j) * kTile, b);
                    kg_last = g;
                }
                // W_hi / W_lo (row-major, MN-major operands) into K stages freed by
                // S_{n-3} / S_{n-2} of this tile
                const int wst_hi = wst_hi_of(base), wst_lo = wst_lo_of(base);
                if (inter && ok && n >= 3)
                    ok = mbar_wait(&bars[B_KEMPTY + wst_hi], ((base + n - 3) / kKStages) & 1, abort_word, a.flags,
                                   a.wait_ns);
                if (inter && ok && n >= 2)
                    ok = mbar_wait(&bars[B_KEMPTY + wst_lo], ((base + n - 2) / kKStages) & 1, abort_word, a.flags,
                                   a.wait_ns);
                // W comes from the prep kernel, which may still be running when this
                // grid starts (programmatic dependent launch): wait for it here
                if (inter) pdl_wait_primary();
                if (inter && ok) {
                    mbar_expect_tx(&bars[B_W], 2 * kTileBytes);
                    tma_load_3d(sb + K0 + wst_hi * kTileBytes, &tm_w, &bars[B_W], 0, 0, bh);
                    tma_load_3d(sb + K0 + wst_hi * kTileBytes + kHalf, &tm_w, &bars[B_W], 64, 0, bh);
                    tma_load_3d(sb + K0 + wst_lo * kTileBytes, &tm_w, &bars[B_W], 0, 0, nbh + bh);
                    tma_load_3d(sb + K0 + wst_lo * kTileBytes + kHalf, &tm_w, &bars[B_W], 64, 0, nbh + bh);
                    w_last = t;
                }
            }

        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer
        // S_g = Q K_j^T into S buffer g&1 (both operands from shared memory);
        // S_{g+2} reuses the buffer as soon as the softmax has S_g in registers,
        // so scores run a tile ahead.  O += P_g V_j once P_g is in its TMEM
        // buffer; the softmax writes P_{g+1} into the other buffer meanwhile.
        // The next query tile's first two score products wait until this tile's
        // epilogue has read O and O_inter (which sits in one of the S buffers)
        // and the next Q has landed.
        if (lane == 0) {
            constexpr uint32_t ID_KK = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t ID_KMN = idesc_bf16(128, 128, 0, 1);
            // descriptors of the first K stage (K-major and, for W, MN-major) and of
            // the first V stage; a stage's descriptor is this plus its offset / 16
            const uint64_t dQ = kmajor_desc(sb + Q, 0), dK = kmajor_desc(sb + K0, 0), dW = mnmajor_desc(sb + K0, 0),
                           dV = mnmajor_desc(sb + V0, 0);
            constexpr uint64_t kStage = kTileBytes >> 4;
            bool ok = true;
            for (int t = 0; t < nt && ok; ++t) {
                const int base = t * n;
                // the tile's first two score products
                if (t > 0 && !(ok = mbar_wait(&bars[B_OFREE], (t - 1) & 1, abort_word, a.flags, a.wait_ns))) break;
                if (!(ok = mbar_wait(&bars[B_Q], t & 1, abort_word, a.flags, a.wait_ns))) break;
                for (int g = base; g < base + 2 && g < base + n && ok; ++g) {
                    const int ks = g % kKStages;
                    if (!(ok = mbar_wait(&bars[B_KFULL + ks], (g / kKStages) & 1, abort_word, a.flags, a.wait_ns)))
                        break;
                    tc_fence_after();
                    mma8_ss<false>(tS0 + (g & 1) * 128, dQ, dK + ks * kStage, ID_KK, 0);
                    mma_commit(&bars[B_SFULL + (g & 1)]);
                    mma_commit(&bars[B_KEMPTY + ks]);
                }
                for (int j = 0; j < n && ok; ++j) {
                    const int g = base + j, sbuf = g & 1;
                    if (j + 2 < n) {
                        const int ks = (g + 2) % kKStages;
                        if (!(ok = mbar_wait(&bars[B_SREAD + sbuf], (g >> 1) & 1, abort_word, a.flags, a.wait_ns)))
                            break;
                        if (!(ok = mbar_wait(&bars[B_KFULL + ks], ((g + 2) / kKStages) & 1, abort_word, a.flags,
                                             a.wait_ns)))
                            break;
                        tc_fence_after();
                        mma8_ss<false>(tS0 + sbuf * 128, dQ, dK + ks * kStage, ID_KK, 0);
                        mma_commit(&bars[B_SFULL + sbuf]);
                        mma_commit(&bars[B_KEMPTY + ks]);
                    }
                    if (inter && j == (n >= 2 ? n - 2 : 0)) {
                        // O_inter = Q W_hi + Q W_lo into the S buffer the tile's last
                        // key tile does not use (free once the softmax has S of key
                        // tile n-2 in registers; unused when n == 1), run while the
                        // softmax works on the last two tiles
                        if (n >= 2 && !(ok = mbar_wait(&bars[B_SREAD + ((base + n) & 1)], ((base + n - 2) >> 1) & 1,
                                                       abort_word, a.flags, a.wait_ns)))
                            break;
                        if (!(ok = mbar_wait(&bars[B_W], t & 1, abort_word, a.flags, a.wait_ns))) break;
                        tc_fence_after();
                        mma8_ss<true>(tOI_of(base), dQ, dW + wst_hi_of(base) * kStage, ID_KMN, 0);
                        mma8_ss<true>(tOI_of(base), dQ, dW + wst_lo_of(base) * kStage, ID_KMN, 1);
                        mma_commit(&bars[B_OIDONE]);
                    }
                    const int vs = g % kVStages;
                    if (!(ok = mbar_wait(&bars[B_PFULL + (g & 1)], (g >> 1) & 1, abort_word, a.flags, a.wait_ns)))
                        break;
                    if (!(ok = mbar_wait(&bars[B_VFULL + vs], (g / kVStages) & 1, abort_word, a.flags, a.wait_ns)))
                        break;
                        mma8_ts<true>(tO, tP + (g & 1) * 64, dV + vs * kStage, ID_KMN, j > 0);
                    mma_commit(&bars[B_PVDONE + (g & 1)]);
                    mma_commit(&bars[B_VEMPTY + vs]);
                }
            }
            // drain: every MMA issued so far completes before TMEM is released
            mma_commit(&bars[B_DRAIN]);
            uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&bars[B_DRAIN]), 0) && globaltimer_ns() - t0 < a.wait_ns) {
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax + epilogue
        // Warps w and w+4 share query rows 32(w&3)..+31 (TMEM lanes); warp w>>2
        // takes score and output columns 64(w>>2)..+63, so two softmax warps
        // per SM sub-partition interleave their exponentials.  S_j is released
        // (SREAD) as soon as it is in registers, so S_{j+2} is computed while
        // this tile is exponentiated, and S_{j+1} is loaded before P_j is
        // handed to the MMA warp.
        //
        // Offset: exponents are taken against a running offset m (log2 units)
        // that is the row max of the first tile and moves only when a tile's
        // partial sum over a half leaves [0, 2^63): the tile is then redone
        // against the row's max and O, l are rescaled.  Every value stays
        // finite, P <= 2^63, and the result is the same softmax (the offset
        // cancels in O / l).
        //
        // The two warps of a pair exchange a code per row and tile (0: a wait
        // failed, 1: ok, 2: offset too low) at their pair barrier and take the
        // same path from it; a warp whose wait failed keeps arriving at the
        // pair barriers to the end, so neither warp ever waits for the other
        // without a partner.
        const int g = warp & 3, hf = warp >> 2;
        const int r = g * 32 + lane;
        const int pair_bar = 1 + g;
        const uint32_t lrow = (uint32_t)(g * 32) << 16;
        const uint32_t cs = hf * 64;
        float* xch = (float*)(smem + XCH);
        uint8_t* xfl = smem + XFL;
        const int mine = hf * 128 + r, theirs = (hf ^ 1) * 128 + r;  // + parity * 256
        const float scale = a.sm_scale_log2;
        float m = 0.f, l = 0.f;
        float A = 0.f;  // kEnt: sum of p (y - m) over this half of the row
        bool ok = true;
        for (int tq = 0; tq < nt; ++tq) {
            const int base = tq * n, q0t = q0_of(tq);
            m = 0.f;
            l = 0.f;
            A = 0.f;
            float x[64];  // this tile's scores (dead in the epilogue)
            ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars[B_SFULL + (base & 1)], (base >> 1) & 1, abort_word,
                                                         a.flags, a.wait_ns));
            if (ok) {
                tc_fence_after();
                const uint32_t src = tS0 + (base & 1) * 128 + lrow + cs;
                tmem_ld32(src, x);
                tmem_ld32(src + 32, x + 32);
            }
            for (int j = 0; j < n; ++j) {
                const int gs = base + j, s = gs & 1;
                const bool w_ok = ok;
                uint32_t pk[32];
                float lt = 0.f;
                if (w_ok) {
                    tmem_ld_wait();
                    tc_fence_before();
                    mbar_arrive(&bars[B_SREAD + s]);  // S_j is in registers: S_{j+2} may overwrite it
                    const int valid = a.T_kv - ktile(j) * kTile - (int)cs;
                    if (valid < 64) {
#pragma unroll
                        for (int c = 0; c < 64; ++c)
                            if (c >= valid) x[c] = -INFINITY;
                    }
                }
                if (j == 0) {
                    // the first tile's row max over both halves sets the offset
                    const float hm = w_ok ? row_max<64>(x) : -INFINITY;
                    xch[mine] = hm;
                    named_bar_sync(pair_bar, 64);
                    m = fmaxf(hm, xch[theirs]) * scale;
                }
                bool redo_h = false;
                float At = 0.f;
                if (w_ok) {
                    lt = kEnt ? exp_scores_ent<64>(x, scale, -m, pk, &At) : exp_scores<64>(x, scale, -m, pk);
                    redo_h = !(lt < 9.2233720e18f);  // >= 2^63, inf or NaN
                }
                xfl[s * 256 + mine] = w_ok ? (redo_h ? 2 : 1) : 0;
                named_bar_sync(pair_bar, 64);
                const uint8_t pc = xfl[s * 256 + theirs];
                ok = __all_sync(0xffffffffu, w_ok && pc != 0);  // the same in both warps of the pair
                const bool redo = ok && (redo_h || pc == 2);
                const bool any_redo = __any_sync(0xffffffffu, redo);
                float f = 1.0f, dm = 0.f;
                if (any_redo) {
                    // the offset is too low for this tile (or a score is not finite):
                    // move it to the row's max and redo P_j; O is rescaled below
                    const float hm = redo ? row_max<64>(x) * scale : -INFINITY;
                    xch[s * 256 + mine] = hm;
                    named_bar_sync(pair_bar, 64);
                    if (redo) {
                        const float mn = fmaxf(m, fmaxf(hm, xch[s * 256 + theirs]));
                        f = ex2(m - mn);
                        dm = mn - m;
                        m = mn;
                    }
                    lt = kEnt ? exp_scores_ent<64>(x, scale, -m, pk, &At) : exp_scores<64>(x, scale, -m, pk);
                }
                if (!ok) continue;  // keep arriving at the pair barriers until the loop ends
                // sum p (y - m) against the moved offset: f (A - dm l) (p scales by f)
                if (kEnt) A = fmaf(f, A - dm * l, At);
                l = fmaf(l, f, lt);
                // P buffer gs & 1 is free once the value product two steps back is
                // done; a rescale of O also waits for the previous step's
                if (gs >= 2) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PVDONE + (gs & 1)], ((gs - 2) >> 1) & 1, abort_word,
                                                           a.flags, a.wait_ns));
                    if (!ok) continue;
                    tc_fence_after();
                }
                if (any_redo && j > 0) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PVDONE + ((gs - 1) & 1)], ((gs - 1) >> 1) & 1,
                                                           abort_word, a.flags, a.wait_ns));
                    if (!ok) continue;
                    tc_fence_after();
                }
                if (any_redo && j > 0) {
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
                tmem_st32u(tP + (gs & 1) * 64 + lrow + hf * 32, pk);
                // this half of S_{j+1} into registers while P_j is being stored
                if (j + 1 < n) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL + (s ^ 1)], ((gs + 1) >> 1) & 1, abort_word,
                                                           a.flags, a.wait_ns));
                    if (ok) {
                        tc_fence_after();
                        const uint32_t src = tS0 + (s ^ 1) * 128 + lrow + cs;
                        tmem_ld32(src, x);
                        tmem_ld32(src + 32, x + 32);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                if (ok) mbar_arrive(&bars[B_PFULL + (gs & 1)]);
            }
            // epilogue: out = O / l + O_inter for this half of the row
            if (ok) tmem_ld_wait();
            const int gl = base + n - 1;  // the tile's last step
            bool e_ok = ok && mbar_wait(&bars[B_PVDONE + (gl & 1)], (gl >> 1) & 1, abort_word, a.flags, a.wait_ns);
            e_ok = __all_sync(0xffffffffu,
                              e_ok && (!inter || mbar_wait(&bars[B_OIDONE], tq & 1, abort_word, a.flags, a.wait_ns)));
            // row sum over the two halves (slot parity of the step after the last:
            // its last readers passed the pair barrier of the tile's last step)
            const int es = ((gl + 1) & 1) * 256;
            xch[es + mine] = l;
            xfl[es + mine] = e_ok ? 1 : 0;
            // kEnt: the halves' sums of p (y - m) through the K stage of the last
            // step (no product reads it any more; W lives in the stages of the
            // steps two and three back)
            float* xa = reinterpret_cast<float*>(smem + K0 + (gl % kKStages) * kTileBytes);
            if (kEnt) xa[mine] = A;
            named_bar_sync(pair_bar, 64);
            const bool both = __all_sync(0xffffffffu, e_ok && xfl[es + theirs] != 0);
            if (both) {
                tc_fence_after();
                const float lrow_sum = l + xch[es + theirs];
                const float inv_l = 1.0f / lrow_sum;  // commutative: the same in both halves
                if (kEnt && hf == 0 && q0t + r < T) {
                    // entropy (nats) of the row's softmax: ln l - ln 2 * sum p (y - m) / l
                    const float at = A + xa[theirs];
                    a.ent_out[(size_t)bh * T + q0t + r] = logf(lrow_sum) - 0.69314718f * at * inv_l;
                }
                // out = a O_intra + O_inter (the inter gain c is folded into W); a = 1 without a mix
                const float inv_out = a.mix ? inv_l * a.mix[bh * 2] : inv_l;
                const int t = q0t + r;
                const size_t row = (((size_t)b * T + t) * a.H + h) * 128 + cs;
                if constexpr (kMulti) {
                    // in two halves of 32 columns (fewer live registers); O and O_inter
                    // are free for the next query tile once both halves are read
#pragma unroll 1
                    for (int c = 0; c < 64; c += 32) {
                        float o[32], e[32];
                        tmem_ld32(tO + lrow + cs + c, o);
                        if (inter) {
                            tmem_ld32(tOI_of(base) + lrow + cs + c, e);
                        } else if (a.oi_ext && t < T) {
                            // token-level access: the read comes from the token-level kernels
                            const float4* src = reinterpret_cast<const float4*>(a.oi_ext + row + c);
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float4 v = src[q];
                                e[4 * q] = v.x;
                                e[4 * q + 1] = v.y;
                                e[4 * q + 2] = v.z;
                                e[4 * q + 3] = v.w;
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 32; ++q) e[q] = 0.f;
                        }
                        tmem_ld_wait();
                        if (c == 32) {
                            tc_fence_before();
                            mbar_arrive(&bars[B_OFREE]);
                        }
                        if (a.out) {
                            // bf16 half-row into box hf of the (free) Q buffer, 128B-swizzled
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                uint4 w;
                                w.x = pack_bf16(o[8 * q + 0] * inv_out + e[8 * q + 0], o[8 * q + 1] * inv_out + e[8 * q + 1]);
                                w.y = pack_bf16(o[8 * q + 2] * inv_out + e[8 * q + 2], o[8 * q + 3] * inv_out + e[8 * q + 3]);
                                w.z = pack_bf16(o[8 * q + 4] * inv_out + e[8 * q + 4], o[8 * q + 5] * inv_out + e[8 * q + 5]);
                                w.w = pack_bf16(o[8 * q + 6] * inv_out + e[8 * q + 6], o[8 * q + 7] * inv_out + e[8 * q + 7]);
                                *reinterpret_cast<uint4*>(smem + Q + hf * kHalf + sw128_offset(r, c / 8 + q)) = w;
                            }
                        }
                        if (a.out_intra && t < T) {
                            float4* di = reinterpret_cast<float4*>(a.out_intra + row + c);
                            float4* de = reinterpret_cast<float4*>(a.out_inter + row + c);
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                di[q] = make_float4(o[4 * q] * inv_l, o[4 * q + 1] * inv_l, o[4 * q + 2] * inv_l,
                                                    o[4 * q + 3] * inv_l);
                                de[q] = make_float4(e[4 * q], e[4 * q + 1], e[4 * q + 2], e[4 * q + 3]);
                            }
                        }
                    }
                    if (a.out) fence_async_smem();
                } else {
                    // the whole half-row at once (one TMEM round trip)
                    float o[64], e[64];
                    tmem_ld32(tO + lrow + cs, o);
                    tmem_ld32(tO + lrow + cs + 32, o + 32);
                    if (inter) {
                        tmem_ld32(tOI_of(base) + lrow + cs, e);
                        tmem_ld32(tOI_of(base) + lrow + cs + 32, e + 32);
                    } else if (a.oi_ext && t < T) {
                        // token-level access: the read comes from the token-level kernels
                        const float4* src = reinterpret_cast<const float4*>(a.oi_ext + row);
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const float4 v = src[q];
                            e[4 * q] = v.x;
                            e[4 * q + 1] = v.y;
                            e[4 * q + 2] = v.z;
                            e[4 * q + 3] = v.w;
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 64; ++q) e[q] = 0.f;
                    }
                    tmem_ld_wait();
                    if (a.out) {
                        // bf16 half-row into box hf of the (free) Q buffer, 128B-swizzled
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            uint4 w;
                            w.x = pack_bf16(o[8 * q + 0] * inv_out + e[8 * q + 0], o[8 * q + 1] * inv_out + e[8 * q + 1]);
                            w.y = pack_bf16(o[8 * q + 2] * inv_out + e[8 * q + 2], o[8 * q + 3] * inv_out + e[8 * q + 3]);
                            w.z = pack_bf16(o[8 * q + 4] * inv_out + e[8 * q + 4], o[8 * q + 5] * inv_out + e[8 * q + 5]);
                            w.w = pack_bf16(o[8 * q + 6] * inv_out + e[8 * q + 6], o[8 * q + 7] * inv_out + e[8 * q + 7]);
                            *reinterpret_cast<uint4*>(smem + Q + hf * kHalf + sw128_offset(r, q)) = w;
                        }
                        fence_async_smem();
                    }
                    if (a.out_intra && t < T) {
                        float4* di = reinterpret_cast<float4*>(a.out_intra + row);
                        float4* de = reinterpret_cast<float4*>(a.out_inter + row);
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            di[q] = make_float4(o[4 * q] * inv_l, o[4 * q + 1] * inv_l, o[4 * q + 2] * inv_l,
                                                o[4 * q + 3] * inv_l);
                            de[q] = make_float4(e[4 * q], e[4 * q + 1], e[4 * q + 2], e[4 * q + 3]);
                        }
                    }
                }
            } else if (kMulti) {
                mbar_arrive(&bars[B_OFREE]);
            }
            // every softmax warp reaches this barrier (no early exit); the tile is
            // stored only if all eight wrote their half-rows
            if (!both && lane == 0) *epi_bad = 1;
            named_bar_sync(5, kSoftmaxThreads);
            if (a.out && threadIdx.x == 0 && *epi_bad == 0) {
                // rows past T are clipped by the tensor map
                tma_store_3d(&tm_o, sb + Q, h * 128, q0t, b);
                tma_store_3d(&tm_o, sb + Q + kHalf, h * 128 + 64, q0t, b);
                bulk_commit_group();
                bulk_wait_read_all();
            }
            // the Q buffer may take the next query tile
            if (kMulti && threadIdx.x == 0) mbar_arrive(&bars[B_QFREE]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // every load a producer issued has landed before the block ends (in a normal
    // run each phase below has long completed; after a wait gave up, some loads
    // were never waited for): the last one on each barrier, bounded (no later
    // load completes a phase of the same barrier)
    if (threadIdx.x == kLoadVWarp * 32) {
        for (int g = vg_last >= kVStages ? vg_last - kVStages + 1 : 0; g <= vg_last; ++g)
            mbar_drain(&bars[B_VFULL + g % kVStages], (g / kVStages) & 1, a.wait_ns);
    } else if (threadIdx.x == kLoadWarp * 32) {
        for (int g = kg_last >= kKStages ? kg_last - kKStages + 1 : 0; g <= kg_last; ++g)
            mbar_drain(&bars[B_KFULL + g % kKStages], (g / kKStages) & 1, a.wait_ns);
        mbar_drain(&bars[B_Q], q_last & 1, a.wait_ns);
        if (w_last >= 0) mbar_drain(&bars[B_W], w_last & 1, a.wait_ns);
    }
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}


}  // namespace tc
}  // namespace hyb
