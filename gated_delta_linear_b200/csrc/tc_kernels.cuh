// tc_kernels.cuh -- tensor-core (tcgen05 / TMEM / TMA) kernels of the hybrid
// layer for bf16 I/O and d = 128 on sm_100a.
//
// Source: "Technical summary: Attend Locally, Remember Linearly (ARL2)",
// gist.science/ar/paper/2605.16579, §2.1 (intra-frame softmax branch,
// inter-frame read O_inter = Q' S_{N-1}, gated delta update) and §2.2
// (frame-level access: all tokens read the pre-update state).
//
// intra_frame_attention: one CTA per (128-query tile, head, batch), 11 warps.
// Warp 8 streams Q and the K ring, warp 10 the V ring, with TMA into
// 128B-swizzled shared memory; warp 9 issues the tcgen05 MMAs; warps 0-7 run
// the online softmax, a query row per pair of threads (warps w and w+4, 64
// scores each in registers).  Near the end of the key loop the Q tile is
// multiplied by W = phi_q^T S_{N-1} (a two-term bf16 split W_hi + W_lo, row
// major: an MN-major B operand), so the inter-frame read lands in TMEM next to
// the softmax accumulator and the epilogue writes out = O_intra + O_inter once.
//   TMEM columns: [0,128) S buffer 0, [128,256) S buffer 1, [256,384) O,
//                 [384,448) Q, [448,512) P (bf16, two per 32-bit column: the
//                 A operands of S = Q K^T and O += P V).  Q is copied from
//                 shared memory into TMEM once; as soon as the softmax has S_j
//                 in registers the MMA warp issues S_{j+2} into its buffer, so
//                 scores run a tile ahead of the softmax, and the softmax loads
//                 S_{j+1} while it hands P_j over.
//   Softmax: exponents against a running offset (the first tile's row max),
//                 moved only when a tile's partial sum over a half row leaves
//                 [0, 2^63); all exponentials on the MUFU pipe.
//   Shared memory: Q 32 KB | K 3 x 32 KB | V 3 x 32 KB.  Near the end W_hi
//                 and W_lo take the K stages of key tiles n-3 and n-2 (unused
//                 stages when n < 3) and O_inter = Q W_hi + Q W_lo goes to the
//                 S buffer the last tile does not use while the softmax works
//                 on the last two tiles; the bf16 output tile is assembled in
//                 the Q buffer and written with two TMA stores.
//   Every CTA signals at entry that the next kernel (the delta update, which
//   reads none of this kernel's outputs) may start on idle SMs.
//
// delta_update: one cluster per (head, batch), one CTA per token split.  Per
// 128-token tile: K~ = K phi_k^T on the tensor core, row L2-normalisation and
// beta in registers, then G += (beta K')^T K' and P += (beta K')^T V as
// MN-major contractions over the tokens, with beta K' and K' split into bf16
// hi + lo (G takes hi*hi + hi*lo + lo*hi, P takes hi*V + lo*V; V is exact in
// bf16); the splits are then reduced through distributed shared memory and
// the update is applied in fp32 (see the kernel's comment).
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace hyb {
namespace tc {

using namespace sm100;

constexpr int kTile = 128;
constexpr uint32_t kTileBytes = 128 * 128 * 2;  // one 128 x 128 bf16 tile
constexpr uint32_t kHalf = kTileBytes / 2;      // one 128 x 64 TMA box
constexpr int kMaxClusterRanks = 8;             // token splits per (b, h) in the update

// ============================================================== attention
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
       B_SREAD = 17, B_QTM = 19, B_PFULL = 20, B_PVDONE = 21, B_COUNT = 22 };
static_assert(B_COUNT * 8 + 8 <= 256, "barrier block");
}  // namespace attn

// K-major operand, 128 rows x 128 bf16 stored as two 64-column swizzled boxes:
// descriptor of the 16-column slice kk (0..7).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kk) {
    return sdesc_sw128(base + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
}
// MN-major operand with the same storage (rows = K index): slice kk covers K rows 16kk..16kk+15.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, int kk) {
    return sdesc_sw128(base + kk * 2048, kHalf, 1024);
}

// Max of N scores (fmaxf: NaN entries are skipped).
template <int N>
__device__ __forceinline__ float row_max(const float* x) {
    float m8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) m8[k] = x[k];
#pragma unroll
    for (int c = 8; c < N; ++c) m8[c & 7] = fmaxf(m8[c & 7], x[c]);
    return fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
}

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
    const int qt_ = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int T = a.T;
    const int q0 = qt_ * kTile;
    const int n = (a.T_kv + kTile - 1) / kTile;  // key tiles
    const bool inter = a.inter != 0;             // add O_inter = Q W (hybrid layer)
    const int bh = b * a.H + h;
    // K stages that receive W_hi / W_lo at the end (free once the scores of key
    // tiles n-3 / n-2 are computed; stages no tile uses when n is small)
    const int wst_hi = n >= 3 ? (n - 3) % kKStages : 2;
    const int wst_lo = n >= 2 ? (n - 2) % kKStages : 1;

    if (threadIdx.x == kLoadWarp * 32) {
        // the producer initialises the barriers and starts the first loads
        // before the block synchronises (the loads land on its own barriers)
        for (int i = 0; i < B_COUNT; ++i)
            mbar_init(&bars[i],
                      (i == B_PFULL || i == B_QTM || i == B_SREAD || i == B_SREAD + 1) ? kSoftmaxThreads : 1);
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
            tma_load_3d(sb + K0 + j * kTileBytes, &tm_k, &bars[B_KFULL + j], xh, j * kTile, b);
            tma_load_3d(sb + K0 + j * kTileBytes + kHalf, &tm_k, &bars[B_KFULL + j], xh + 64, j * kTile, b);
        }
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // S buffers 0 / 1, O, Q and P as bf16 pairs (the A operands of the score
    // and value products)
    const uint32_t tS0 = tmem, tO = tmem + 256, tQ = tmem + 384, tP = tmem + 448;
    const uint32_t tOI = tS0 + (n & 1) * 128;  // the S buffer the last tile does not use

    if (warp == kLoadVWarp) {
        // ------------------------------------------------ TMA producer: V ring
        if (lane == 0) {
            tma_prefetch_desc(&tm_v);
            const int xh = h * 128;
            for (int j = 0; j < n; ++j) {
                const int vs = j % kVStages;
                if (j >= kVStages &&
                    !mbar_wait(&bars[B_VEMPTY + vs], ((j / kVStages) + 1) & 1, abort_word, a.flags))
                    break;
                mbar_expect_tx(&bars[B_VFULL + vs], kTileBytes);
                tma_load_3d(sb + V0 + vs * kTileBytes, &tm_v, &bars[B_VFULL + vs], xh, j * kTile, b);
                tma_load_3d(sb + V0 + vs * kTileBytes + kHalf, &tm_v, &bars[B_VFULL + vs], xh + 64, j * kTile, b);
            }
        }
        __syncwarp();
    } else if (warp == kLoadWarp) {
        // ------------------------------------------------ TMA producer: Q, K ring, W
        // (its own warp, so K tiles run ahead of the V ring's waits)
        if (lane == 0) {
            tma_prefetch_desc(&tm_w);
            const int xh = h * 128;
            bool ok = true;
            for (int j = kKStages; j < n && ok; ++j) {  // Q and K_0..K_2 were issued at entry
                const int ks = j % kKStages;
                if (!(ok = mbar_wait(&bars[B_KEMPTY + ks], ((j / kKStages) + 1) & 1, abort_word, a.flags))) break;
                mbar_expect_tx(&bars[B_KFULL + ks], kTileBytes);
                tma_load_3d(sb + K0 + ks * kTileBytes, &tm_k, &bars[B_KFULL + ks], xh, j * kTile, b);
                tma_load_3d(sb + K0 + ks * kTileBytes + kHalf, &tm_k, &bars[B_KFULL + ks], xh + 64, j * kTile, b);
            }
            // W_hi / W_lo (row-major, MN-major operands) into K stages freed by S_{n-3} / S_{n-2}
            const int nbh = a.B * a.H;
            if (inter && ok && n >= 3)
                ok = mbar_wait(&bars[B_KEMPTY + wst_hi], ((n - 3) / kKStages) & 1, abort_word, a.flags);
            if (inter && ok && n >= 2)
                ok = mbar_wait(&bars[B_KEMPTY + wst_lo], ((n - 2) / kKStages) & 1, abort_word, a.flags);
            // W comes from the prep kernel, which may still be running when this
            // grid starts (programmatic dependent launch): wait for it here
            if (inter) pdl_wait_primary();
            if (inter && ok) {
                mbar_expect_tx(&bars[B_W], 2 * kTileBytes);
                tma_load_3d(sb + K0 + wst_hi * kTileBytes, &tm_w, &bars[B_W], 0, 0, bh);
                tma_load_3d(sb + K0 + wst_hi * kTileBytes + kHalf, &tm_w, &bars[B_W], 64, 0, bh);
                tma_load_3d(sb + K0 + wst_lo * kTileBytes, &tm_w, &bars[B_W], 0, 0, nbh + bh);
                tma_load_3d(sb + K0 + wst_lo * kTileBytes + kHalf, &tm_w, &bars[B_W], 64, 0, nbh + bh);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer
        // S_j = Q K_j^T into S buffer j&1 (A = Q from TMEM); S_{j+2} reuses the
        // buffer as soon as the softmax has S_j in registers, so scores run a
        // tile ahead.  O += P_j V_j once P_j is in TMEM.
        if (lane == 0) {
            constexpr uint32_t ID_KK = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t ID_KMN = idesc_bf16(128, 128, 0, 1);
            // S_0 and S_1 take Q from shared memory (no wait for its copy into TMEM)
            bool ok = mbar_wait(&bars[B_Q], 0, abort_word, a.flags);
            bool q_in_tmem = false;
            for (int j = 0; j < 2 && j < n && ok; ++j) {
                if (!(ok = mbar_wait(&bars[B_KFULL + j], 0, abort_word, a.flags))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tS0 + j * 128, kmajor_desc(sb + Q, kk), kmajor_desc(sb + K0 + j * kTileBytes, kk), ID_KK,
                             kk > 0);
                mma_commit(&bars[B_SFULL + j]);
                mma_commit(&bars[B_KEMPTY + j]);
            }
            for (int j = 0; j < n && ok; ++j) {
                const int sbuf = j & 1;
                if (j + 2 < n) {
                    const int ks = (j + 2) % kKStages;
                    if (!q_in_tmem && !(ok = q_in_tmem = mbar_wait(&bars[B_QTM], 0, abort_word, a.flags))) break;
                    if (!(ok = mbar_wait(&bars[B_SREAD + sbuf], (j >> 1) & 1, abort_word, a.flags))) break;
                    if (!(ok = mbar_wait(&bars[B_KFULL + ks], ((j + 2) / kKStages) & 1, abort_word, a.flags))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tS0 + sbuf * 128, tQ + kk * 8, kmajor_desc(sb + K0 + ks * kTileBytes, kk), ID_KK,
                                    kk > 0);
                    mma_commit(&bars[B_SFULL + sbuf]);
                    mma_commit(&bars[B_KEMPTY + ks]);
                }
                if (inter && j == (n >= 2 ? n - 2 : 0)) {
                    // O_inter = Q W_hi + Q W_lo into S buffer n&1 (free once the
                    // softmax has S_{n-2} in registers; unused when n == 1), run
                    // while the softmax works on the last two tiles
                    if (!q_in_tmem && !(ok = q_in_tmem = mbar_wait(&bars[B_QTM], 0, abort_word, a.flags))) break;
                    if (n >= 2 &&
                        !(ok = mbar_wait(&bars[B_SREAD + (n & 1)], ((n - 2) >> 1) & 1, abort_word, a.flags)))
                        break;
                    if (!(ok = mbar_wait(&bars[B_W], 0, abort_word, a.flags))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tOI, tQ + kk * 8, mnmajor_desc(sb + K0 + wst_hi * kTileBytes, kk), ID_KMN, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tOI, tQ + kk * 8, mnmajor_desc(sb + K0 + wst_lo * kTileBytes, kk), ID_KMN, 1);
                    mma_commit(&bars[B_OIDONE]);
                }
                const int vs = j % kVStages;
                if (!(ok = mbar_wait(&bars[B_PFULL], j & 1, abort_word, a.flags))) break;
                if (!(ok = mbar_wait(&bars[B_VFULL + vs], (j / kVStages) & 1, abort_word, a.flags))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tO, tP + kk * 8, mnmajor_desc(sb + V0 + vs * kTileBytes, kk), ID_KMN, (j > 0 || kk > 0));
                mma_commit(&bars[B_PVDONE]);
                mma_commit(&bars[B_VEMPTY + vs]);
            }
            // drain: every MMA issued so far completes before TMEM is released
            mma_commit(&bars[B_Q]);
            uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&bars[B_Q]), 1) && globaltimer_ns() - t0 < kWaitNs) {
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
        float x[64];
        // this half of Q row r (128B-swizzled in shared memory) into TMEM as bf16 pairs
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_Q], 0, abort_word, a.flags));
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
            tc_fence_before();
            mbar_arrive(&bars[B_QTM]);
        }
        ok = ok && __all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL], 0, abort_word, a.flags));
        if (ok) {
            tc_fence_after();
            tmem_ld32(tS0 + lrow + cs, x);
            tmem_ld32(tS0 + lrow + cs + 32, x + 32);
        }
        for (int j = 0; j < n; ++j) {
            const int s = j & 1;
            const bool w_ok = ok;
            uint32_t pk[32];
            float lt = 0.f;
            if (w_ok) {
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&bars[B_SREAD + s]);  // S_j is in registers: S_{j+2} may overwrite it
                const int valid = a.T_kv - j * kTile - (int)cs;
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
            if (w_ok) {
                lt = exp_scores<64>(x, scale, -m, pk);
                redo_h = !(lt < 9.2233720e18f);  // >= 2^63, inf or NaN
            }
            xfl[s * 256 + mine] = w_ok ? (redo_h ? 2 : 1) : 0;
            named_bar_sync(pair_bar, 64);
            const uint8_t pc = xfl[s * 256 + theirs];
            ok = __all_sync(0xffffffffu, w_ok && pc != 0);  // the same in both warps of the pair
            const bool redo = ok && (redo_h || pc == 2);
            const bool any_redo = __any_sync(0xffffffffu, redo);
            float f = 1.0f;
            if (any_redo) {
                // the offset is too low for this tile (or a score is not finite):
                // move it to the row's max and redo P_j; O is rescaled below
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
            if (!ok) continue;  // keep arriving at the pair barriers until the loop ends
            l = fmaf(l, f, lt);
            // the P buffer (and O) are free once P_{j-1} V_{j-1} is done
            if (j > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PVDONE], (j - 1) & 1, abort_word, a.flags));
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
            tmem_st32u(tP + lrow + hf * 32, pk);
            // this half of S_{j+1} into registers while P_j is being stored
            if (j + 1 < n) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL + (s ^ 1)], ((j + 1) >> 1) & 1, abort_word,
                                                       a.flags));
                if (ok) {
                    tc_fence_after();
                    const uint32_t src = tS0 + (s ^ 1) * 128 + lrow + cs;
                    tmem_ld32(src, x);
                    tmem_ld32(src + 32, x + 32);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            if (ok) mbar_arrive(&bars[B_PFULL]);
        }
        // epilogue: out = O / l + O_inter for this half of the row
        if (ok) tmem_ld_wait();
        bool e_ok = ok && mbar_wait(&bars[B_PVDONE], (n - 1) & 1, abort_word, a.flags);
        e_ok = __all_sync(0xffffffffu, e_ok && (!inter || mbar_wait(&bars[B_OIDONE], 0, abort_word, a.flags)));
        // row sum over the two halves (slot parity n&1: its last readers passed
        // the pair barrier of tile n-1)
        xch[(n & 1) * 256 + mine] = l;
        xfl[(n & 1) * 256 + mine] = e_ok ? 1 : 0;
        named_bar_sync(pair_bar, 64);
        const bool both = __all_sync(0xffffffffu, e_ok && xfl[(n & 1) * 256 + theirs] != 0);
        if (both) {
            tc_fence_after();
            const float inv_l = 1.0f / (l + xch[(n & 1) * 256 + theirs]);  // commutative: the same in both halves
            // out = a O_intra + O_inter (the inter gain c is folded into W); a = 1 without a mix
            const float inv_out = a.mix ? inv_l * a.mix[bh * 2] : inv_l;
            const int t = q0 + r;
            const size_t row = (((size_t)b * T + t) * a.H + h) * 128 + cs;
            float o[64], e[64];
            tmem_ld32(tO + lrow + cs, o);
            tmem_ld32(tO + lrow + cs + 32, o + 32);
            if (inter) {
                tmem_ld32(tOI + lrow + cs, e);
                tmem_ld32(tOI + lrow + cs + 32, e + 32);
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
        // every softmax warp reaches this barrier (no early exit); the tile is
        // stored only if all eight wrote their half-rows
        if (!both && lane == 0) *epi_bad = 1;
        named_bar_sync(5, kSoftmaxThreads);
        if (a.out && threadIdx.x == 0 && *epi_bad == 0) {
            // rows past T are clipped by the tensor map
            tma_store_3d(&tm_o, sb + Q, h * 128, q0, b);
            tma_store_3d(&tm_o, sb + Q + kHalf, h * 128 + 64, q0, b);
            bulk_commit_group();
            bulk_wait_read_all();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// ============================================================== delta update
// One cluster of C CTAs per (batch, head); CTA c of the cluster takes token
// split c (a run of 128-token tiles) and accumulates its G_c = (beta K')^T K'
// and P_c = (beta K')^T V in TMEM.  Since the update is linear in the splits,
// every CTA then forms its own contribution Delta_c = P_c phi_v^T - G_c S_{N-1}
// on the tensor core (bf16 hi + lo splits of G_c, P_c and S_{N-1}), and each
// CTA sums one band of rows of Delta over the C CTAs through distributed
// shared memory (fixed order c = 0..C-1, so the result is deterministic):
//   S_N[i][:] = alpha S_{N-1}[i][:] + sum_c Delta_c[i][:]
// with alpha = mean_t sigmoid(g_t).  Every CTA stages S_{N-1} from the state
// buffer before the cluster's first barrier and writes its band after it.  The
// kernel reads only the pass's inputs and the state, never the prep kernel's
// outputs, so it may run alongside the attention kernel.
namespace upd {
// tile loop (1024-aligned 128B-swizzled tiles)
constexpr uint32_t PHI = 0;
constexpr uint32_t KT = PHI + kTileBytes;
constexpr uint32_t VT = KT + kTileBytes;
constexpr uint32_t AH = VT + kTileBytes;
constexpr uint32_t AL = AH + kTileBytes;
constexpr uint32_t KH = AL + kTileBytes;
constexpr uint32_t KL = KH + kTileBytes;
constexpr uint32_t TILES_END = KL + kTileBytes;          // 229,376
// after the tile loop (reuses the tile space)
constexpr uint32_t PHIV = 0;                              // phi_v, K-major B operand (rows j, o contiguous)
constexpr uint32_t SPREV = PHIV + kTileBytes;             // S_{N-1} fp32 [128][128]
constexpr uint32_t SH = SPREV + 128 * 128 * 4;            // S_hi, MN-major B operand (rows m, j contiguous)
constexpr uint32_t SL = SH + kTileBytes;                  // S_lo
constexpr uint32_t RED = SL + kTileBytes;                 // Delta_c fp32 [128][128], 16-byte chunks XOR-swizzled
constexpr uint32_t BAR = TILES_END;                       // barriers, TMEM slot, flags, sums
constexpr uint32_t XSS = BAR + 256;                       // [2 parity][2 halves][128 rows] floats + ok bytes
constexpr uint32_t SMEM = XSS + 2048 + 512;               // 232,192 B
constexpr int kNormThreads = 256;                         // warps 0-7
constexpr int kLoadWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 320;
enum { B_PHI = 0, B_KFULL, B_KFREE, B_VFULL, B_KTFULL, B_OPSFULL, B_OPSFREE, B_PARK, B_DELTA, B_COUNT };
static_assert(RED + 128 * 128 * 4 <= TILES_END, "post-loop buffers exceed the tile space");
// byte offset of float4 chunk q (0..31) of row `row` in RED
__device__ __forceinline__ uint32_t red_off(int row, int q) {
    return (uint32_t)(row * 512 + ((q ^ (row & 7)) << 4));
}
}  // namespace upd

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(remote)
                 : "memory");
    return v;
}

__global__ void __launch_bounds__(upd::kThreads, 1)
    update_kernel(const __grid_constant__ LayerArgs a, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_phik) {
    using namespace upd;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {  // uniform over the grid: every CTA leaves
        if (threadIdx.x == 0) atomicOr(a.flags, FLAG_INTERNAL);
        return;
    }
    const uint32_t sb = smem_u32(smem);
    uint64_t* bars = (uint64_t*)(smem + BAR);
    uint32_t* tmem_slot = (uint32_t*)(bars + B_COUNT);
    volatile int* abort_word = (volatile int*)(tmem_slot + 1);
    float* wsum = (float*)(tmem_slot + 2);  // 10 warp partial sums + alpha
    float* xss = (float*)(smem + XSS);      // row sums of squares exchanged between warp pairs
    uint8_t* xok = smem + XSS + 2048;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y, b = blockIdx.z;
    const int split = (int)cluster_ctarank();
    const int C = (int)cluster_nctarank();
    const int T = a.T;
    const int bh = b * a.H + h;
    const int t_begin = split * a.split_tokens;
    const int t_end = min(T, t_begin + a.split_tokens);
    const int nt = t_end > t_begin ? (t_end - t_begin + kTile - 1) / kTile : 0;
    // this thread's first gate logits (for alpha), loaded now and summed after the tile loop
    const float* gl = a.gate_logits + (size_t)bh * T;
    float g0[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) g0[u] = (threadIdx.x + u * kThreads < T) ? gl[threadIdx.x + u * kThreads] : 0.f;

    if (threadIdx.x == 0) {
        for (int i = 0; i < B_COUNT; ++i) mbar_init(&bars[i], i == B_OPSFULL ? kNormThreads : 1);
        *abort_word = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tKT = tmem, tG = tmem + 128, tP = tmem + 256;

    uint4 pv[8];  // phi_v staging (normalisation warps)
    // ------------------------------------------------------------ tile loop
    if (warp == kLoadWarp) {
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_phik);
            const int xh = h * 128;
            mbar_expect_tx(&bars[B_PHI], kTileBytes);
            tma_load_3d(sb + PHI, &tm_phik, &bars[B_PHI], 0, 0, h);
            tma_load_3d(sb + PHI + kHalf, &tm_phik, &bars[B_PHI], 64, 0, h);
            for (int i = 0; i < nt; ++i) {
                const int t0 = t_begin + i * kTile;
                if (i > 0 && !mbar_wait(&bars[B_KFREE], (i - 1) & 1, abort_word, a.flags)) break;
                mbar_expect_tx(&bars[B_KFULL], kTileBytes);
                tma_load_3d(sb + KT, &tm_k, &bars[B_KFULL], xh, t0, b);
                tma_load_3d(sb + KT + kHalf, &tm_k, &bars[B_KFULL], xh + 64, t0, b);
                if (i > 0 && !mbar_wait(&bars[B_OPSFREE], (i - 1) & 1, abort_word, a.flags)) break;
                mbar_expect_tx(&bars[B_VFULL], kTileBytes);
                tma_load_3d(sb + VT, &tm_v, &bars[B_VFULL], xh, t0, b);
                tma_load_3d(sb + VT + kHalf, &tm_v, &bars[B_VFULL], xh + 64, t0, b);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        if (lane == 0 && nt > 0) {
            constexpr uint32_t ID_KK = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t ID_MNMN = idesc_bf16(128, 128, 1, 1);
            bool ok = mbar_wait(&bars[B_PHI], 0, abort_word, a.flags);
            for (int i = 0; i < nt && ok; ++i) {
                const uint32_t par = i & 1;
                if (!mbar_wait(&bars[B_KFULL], par, abort_word, a.flags)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tKT, kmajor_desc(sb + KT, kk), kmajor_desc(sb + PHI, kk), ID_KK, kk > 0);
                mma_commit(&bars[B_KTFULL]);
                mma_commit(&bars[B_KFREE]);
                if (!mbar_wait(&bars[B_OPSFULL], par, abort_word, a.flags)) break;
                if (!mbar_wait(&bars[B_VFULL], par, abort_word, a.flags)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t acc = (i > 0 || kk > 0);
                    mma_bf16(tG, mnmajor_desc(sb + AH, kk), mnmajor_desc(sb + KH, kk), ID_MNMN, acc);
                    mma_bf16(tG, mnmajor_desc(sb + AH, kk), mnmajor_desc(sb + KL, kk), ID_MNMN, 1);
                    mma_bf16(tG, mnmajor_desc(sb + AL, kk), mnmajor_desc(sb + KH, kk), ID_MNMN, 1);
                    mma_bf16(tP, mnmajor_desc(sb + AH, kk), mnmajor_desc(sb + VT, kk), ID_MNMN, acc);
                    mma_bf16(tP, mnmajor_desc(sb + AL, kk), mnmajor_desc(sb + VT, kk), ID_MNMN, 1);
                }
                mma_commit(&bars[B_OPSFREE]);
            }
            // drain: every MMA issued so far completes before the tile space is reused
            mma_commit(&bars[B_PHI]);
            uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&bars[B_PHI]), 1) && globaltimer_ns() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
    } else {
        // Warps w and w+4 share token rows (TMEM lanes 32(w%4)..+31); warp w/4 = half
        // takes feature columns 64*half..64*half+63.  The pair exchanges its half
        // sums of squares (and wait results) at a named barrier every tile.
        const int half = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const int pair_bar = 1 + (warp & 3);
        const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
        bool ok = true;
        float x[64];
        for (int i = 0; i < nt; ++i) {
            const int s = i & 1;
            // this row's beta logit, loaded before the wait for K~
            const int tok = t_begin + i * kTile + r;
            const bool valid = tok < t_end;
            const float bl = valid ? a.beta_logits[(size_t)bh * T + tok] : 0.f;
            bool w_ok = ok && mbar_wait(&bars[B_KTFULL], i & 1, abort_word, a.flags);
            if (i > 0) w_ok = w_ok && mbar_wait(&bars[B_OPSFREE], (i - 1) & 1, abort_word, a.flags);
            w_ok = __all_sync(0xffffffffu, w_ok);
            float ssh = 0.f;
            if (w_ok) {
                tc_fence_after();
                tmem_ld32(tKT + lrow + half * 64, x);
                tmem_ld32(tKT + lrow + half * 64 + 32, x + 32);
                tmem_ld_wait();
                float ss8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) ss8[k] = 0.f;
#pragma unroll
                for (int c = 0; c < 64; ++c) ss8[c & 7] = fmaf(x[c], x[c], ss8[c & 7]);
                ssh = ((ss8[0] + ss8[1]) + (ss8[2] + ss8[3])) + ((ss8[4] + ss8[5]) + (ss8[6] + ss8[7]));
            }
            xss[(s * 2 + half) * 128 + r] = ssh;
            xok[(s * 2 + half) * 128 + r] = (uint8_t)w_ok;
            named_bar_sync(pair_bar, 64);
            ok = __all_sync(0xffffffffu, w_ok && xok[(s * 2 + (half ^ 1)) * 128 + r]);
            if (!ok) continue;  // keep arriving at the pair barriers until the loop ends
            const float ss = xss[(s * 2 + 0) * 128 + r] + xss[(s * 2 + 1) * 128 + r];
            const float inv = valid ? 1.0f / sqrtf(ss + a.l2_eps) : 0.f;
            const float beta = valid ? sigmoidf_(bl) : 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t ah[4], al[4], kh[4], kl[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int col = c * 8 + 2 * q;
                    const float k0 = x[col] * inv, k1 = x[col + 1] * inv;
                    const float a0 = k0 * beta, a1 = k1 * beta;
                    const __nv_bfloat162 khv = __floats2bfloat162_rn(k0, k1);
                    const __nv_bfloat162 ahv = __floats2bfloat162_rn(a0, a1);
                    kh[q] = *reinterpret_cast<const uint32_t*>(&khv);
                    ah[q] = *reinterpret_cast<const uint32_t*>(&ahv);
                    kl[q] = pack_bf16(k0 - __low2float(khv), k1 - __high2float(khv));
                    al[q] = pack_bf16(a0 - __low2float(ahv), a1 - __high2float(ahv));
                }
                const uint32_t off = half * kHalf + sw128_offset(r, c);
                *reinterpret_cast<uint4*>(smem + AH + off) = make_uint4(ah[0], ah[1], ah[2], ah[3]);
                *reinterpret_cast<uint4*>(smem + AL + off) = make_uint4(al[0], al[1], al[2], al[3]);
                *reinterpret_cast<uint4*>(smem + KH + off) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
                *reinterpret_cast<uint4*>(smem + KL + off) = make_uint4(kl[0], kl[1], kl[2], kl[3]);
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_OPSFULL]);
        }
        // phi_v row r, columns 64 half..+63, loaded while the last products run
        {
            const uint4* src = reinterpret_cast<const uint4*>((const __nv_bfloat16*)a.phi_v +
                                                              (size_t)h * 128 * 128 + (size_t)r * 128 + half * 64);
#pragma unroll
            for (int c = 0; c < 8; ++c) pv[c] = src[c];
        }
        if (ok && nt > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_OPSFREE], (nt - 1) & 1, abort_word, a.flags));
    }
    // ------------------------------------------------------------ Delta_c = P_c phi_v^T - G_c S_{N-1}
    // G_c and P_c (fp32 in TMEM) become bf16 hi + lo A operands in TMEM; S_{N-1}
    // becomes a bf16 hi + lo B operand and phi_v a K-major B operand in shared
    // memory; five MMAs give this split's contribution, which the cluster sums.
    const uint32_t tGH = tmem, tGL = tmem + 64, tD = tmem + 128, tPH = tmem + 384, tPL = tmem + 448;
    tc_fence_before();
    __syncthreads();  // every MMA of the tile loop has completed (or timed out)
    tc_fence_after();
    if (threadIdx.x == kLoadWarp * 32) {
        mbar_expect_tx(&bars[B_PARK], 128 * 128 * 4);
        bulk_load(sb + SPREV, a.state + (size_t)bh * 128 * 128, 128 * 128 * 4, &bars[B_PARK]);
    }
    {
        // alpha: the entry loads, then any further logits (T > 8 x 320), each
        // batch loaded before its sigmoids are taken
        float sg = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (threadIdx.x + u * kThreads < T) sg += sigmoidf_(g0[u]);
        for (int t0 = threadIdx.x + 8 * kThreads; t0 < T; t0 += 8 * kThreads) {
            float g[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) g[u] = (t0 + u * kThreads < T) ? gl[t0 + u * kThreads] : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (t0 + u * kThreads < T) sg += sigmoidf_(g[u]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sg += __shfl_xor_sync(0xffffffffu, sg, o);
        if (lane == 0) wsum[warp] = sg;
    }
    bool park_ok = true;
    if (warp < 8) {
        const int half = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
        // phi_v row `row`, columns 64 half..+63 (loaded during the tile loop), into the K-major B tile
#pragma unroll
        for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(smem + PHIV + half * kHalf + sw128_offset(row, c)) = pv[c];
        // G and P rows `row`, columns 64 half..+63: fp32 -> bf16 hi + lo in TMEM
#pragma unroll
        for (int gp = 0; gp < 2; ++gp) {
            float x[64];
            uint32_t hi[32], lo[32];
            const uint32_t src = (gp == 0 ? tG : tP) + lrow + half * 64;
            if (nt > 0) {
                tmem_ld32(src, x);
                tmem_ld32(src + 32, x + 32);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int q = 0; q < 64; ++q) x[q] = 0.f;
            }
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const __nv_bfloat162 hv = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
                hi[q] = *reinterpret_cast<const uint32_t*>(&hv);
                lo[q] = pack_bf16(x[2 * q] - __low2float(hv), x[2 * q + 1] - __high2float(hv));
            }
            tmem_st32u((gp == 0 ? tGH : tPH) + lrow + half * 32, hi);
            tmem_st32u((gp == 0 ? tGL : tPL) + lrow + half * 32, lo);
        }
        tmem_st_wait();
        // S_{N-1} row `row`, columns 64 half..+63: bf16 hi + lo into the MN-major B tiles
        park_ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PARK], 0, abort_word, a.flags));
        // float4 k of the row half is read in the order (k0 + lane) & 15, so a
        // warp's reads (rows 512 B apart) spread over all 16-byte bank groups
        const float4* Sp4 = reinterpret_cast<const float4*>(smem + SPREV) + row * 32 + half * 16;
#pragma unroll
        for (int k0 = 0; k0 < 16; ++k0) {
            const int k = (k0 + lane) & 15;
            const float4 v = Sp4[k];
            const __nv_bfloat162 h01 = __floats2bfloat162_rn(v.x, v.y);
            const __nv_bfloat162 h23 = __floats2bfloat162_rn(v.z, v.w);
            const uint2 hi = make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
            const uint2 lo = make_uint2(pack_bf16(v.x - __low2float(h01), v.y - __high2float(h01)),
                                        pack_bf16(v.z - __low2float(h23), v.w - __high2float(h23)));
            const uint32_t off = half * kHalf + sw128_offset(row, k >> 1) + (k & 1) * 8;
            *reinterpret_cast<uint2*>(smem + SH + off) = hi;
            *reinterpret_cast<uint2*>(smem + SL + off) = lo;
        }
    } else {
        // S_{N-1} must be in shared memory before any CTA of the cluster passes the
        // first cluster barrier: after it, CTAs write their bands of the state
        park_ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PARK], 0, abort_word, a.flags));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == kMmaWarp * 32) {
        constexpr uint32_t ID_KK = idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t ID_KMN_NEG = idesc_bf16(128, 128, 0, 1) | (1u << 13);  // -A
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ts(tD, tPH + kk * 8, kmajor_desc(sb + PHIV, kk), ID_KK, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ts(tD, tPL + kk * 8, kmajor_desc(sb + PHIV, kk), ID_KK, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ts(tD, tGH + kk * 8, mnmajor_desc(sb + SH, kk), ID_KMN_NEG, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ts(tD, tGH + kk * 8, mnmajor_desc(sb + SL, kk), ID_KMN_NEG, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ts(tD, tGL + kk * 8, mnmajor_desc(sb + SH, kk), ID_KMN_NEG, 1);
        mma_commit(&bars[B_DELTA]);
    }
    if (warp < 8) {
        // Delta_c row `row`, columns 64 half..+63, into shared memory for the cluster
        const int half = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
        const bool d_ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_DELTA], 0, abort_word, a.flags));
        tc_fence_after();
        float v[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            if (d_ok) {
                tmem_ld32(tD + lrow + half * 64 + c * 32, v);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int q = 0; q < 32; ++q) v[q] = 0.f;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4*>(smem + RED + red_off(row, half * 16 + c * 8 + q)) =
                    make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) t += wsum[w];
        wsum[10] = t / (float)T;
    }
    cluster_sync();  // every CTA of the cluster has parked Delta_c and staged S_{N-1}

    // ------------------------------------------------------------ reduce and apply this CTA's band
    // S_N[row] = alpha S_{N-1}[row] + sum_c Delta_c[row], ranks summed in order
    {
        const int band = (128 + C - 1) / C;
        const int r0 = min(128, split * band), r1 = min(128, r0 + band);
        const float alpha = wsum[10];
        const float* Sp = reinterpret_cast<const float*>(smem + SPREV);
        float* S = a.state + (size_t)bh * 128 * 128;
        const int items = (r1 - r0) * 32;
        bool bad = false;
        for (int it = threadIdx.x; it < items && park_ok; it += 2 * kThreads) {
            const int it2 = it + kThreads;
            const bool second = it2 < items;
            const int row0 = r0 + it / 32, q0 = it % 32;
            const int row1 = second ? r0 + it2 / 32 : row0, q1 = second ? it2 % 32 : q0;
            const uint32_t off0 = red_off(row0, q0), off1 = red_off(row1, q1);
            float4 v0[kMaxClusterRanks], v1[kMaxClusterRanks];
#pragma unroll
            for (int c = 0; c < kMaxClusterRanks; ++c)
                if (c < C) {
                    v0[c] = ld_cluster_f4(sb + RED + off0, (uint32_t)c);
                    v1[c] = ld_cluster_f4(sb + RED + off1, (uint32_t)c);
                }
            float4 s0 = *reinterpret_cast<const float4*>(Sp + row0 * 128 + q0 * 4);
            float4 s1 = *reinterpret_cast<const float4*>(Sp + row1 * 128 + q1 * 4);
            s0 = make_float4(alpha * s0.x, alpha * s0.y, alpha * s0.z, alpha * s0.w);
            s1 = make_float4(alpha * s1.x, alpha * s1.y, alpha * s1.z, alpha * s1.w);
#pragma unroll
            for (int c = 0; c < kMaxClusterRanks; ++c)
                if (c < C) {
                    s0.x += v0[c].x; s0.y += v0[c].y; s0.z += v0[c].z; s0.w += v0[c].w;
                    s1.x += v1[c].x; s1.y += v1[c].y; s1.z += v1[c].z; s1.w += v1[c].w;
                }
            *reinterpret_cast<float4*>(S + row0 * 128 + q0 * 4) = s0;
            bad |= !(isfinite(s0.x) && isfinite(s0.y) && isfinite(s0.z) && isfinite(s0.w));
            if (second) {
                *reinterpret_cast<float4*>(S + row1 * 128 + q1 * 4) = s1;
                bad |= !(isfinite(s1.x) && isfinite(s1.y) && isfinite(s1.z) && isfinite(s1.w));
            }
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(a.flags, FLAG_NONFINITE);
    }
    cluster_sync();  // no CTA leaves while another still reads its shared memory
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
    // when launched as a programmatic dependent of the attention kernel, complete
    // only after it: later work in the stream stays ordered after both
    pdl_wait_primary();
}

}  // namespace tc
}  // namespace hyb
