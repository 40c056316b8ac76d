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
// One CTA takes two 128-query tiles (A and B) of one (batch, head) and streams
// the frame's keys and values past both in 128-key blocks:
//   warps 0-3   softmax of tile A, one query row (TMEM lane) per thread;
//   warps 4-7   softmax of tile B;
//   warp 8      TMA producer of Q_A, Q_B, the K ring and, at the end, W;
//   warp 9      the single tcgen05 MMA issuer;
//   warp 10     TMA producer of the V ring.
// The two tiles ping-pong: while the softmax warps of one tile turn its scores
// into probabilities on the MUFU pipe, the tensor pipe runs the other tile's
// O += P V and its next S = Q K^T, so neither pipe waits for the other.
//
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
// P_t (bf16 pairs, the A operand of O_t += P_t V) is written over the first 64
// columns of S_t once the scores are in registers.  MMAs into different
// accumulators are not ordered by the hardware, so S_t(j+1) is issued only
// after O_t += P_t(j) V_j has completed.
//
// Softmax offset: probabilities are 2^(s x - m) with a per-row offset m (the
// first block's row max, in log2 units) that moves only when a block's row sum
// leaves [0, 2^63): then the block is redone against the row's max and O, l
// are rescaled (O_t is idle then: S_t(j) is issued after P_t(j-1) V has
// completed).  The offset cancels in O / l, so this is the same softmax.
//
// Epilogue: after the last block each tile's S buffer is free, and O_inter = Q_t W_hi + Q_t W_lo (W = phi_q^T S_{N-1}, a two-term
// bf16 split written by the prep kernel, loaded into K stages the last score
// products have freed) is computed there; out = a O_t / l + O_inter is rounded
// once to bf16, staged in the tile's Q buffer and written with TMA stores.
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace hyb {
namespace tc {

using namespace sm100;

namespace pp {
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t QA = 0;
constexpr uint32_t QB = QA + kTileBytes;
constexpr uint32_t K0 = QB + kTileBytes;
constexpr uint32_t V0 = K0 + kKStages * kTileBytes;
constexpr uint32_t BAR = V0 + kVStages * kTileBytes;   // 229,376
constexpr uint32_t SMEM = BAR + 256;                    // 229,632 B
constexpr int kThreads = 352;  // 11 warps: up to 184 registers per thread
constexpr int kLoadWarp = 8, kMmaWarp = 9, kLoadVWarp = 10;
enum {
    B_QA = 0, B_QB = 1, B_W = 2, B_KFULL = 3, B_KEMPTY = B_KFULL + kKStages, B_VFULL = B_KEMPTY + kKStages,
    B_VEMPTY = B_VFULL + kVStages, B_SFULL = B_VEMPTY + kVStages, B_PFULL = B_SFULL + 2, B_PVDONE = B_PFULL + 2,
    B_OIDONE = B_PVDONE + 2, B_DRAIN = B_OIDONE + 2, B_TURN = B_DRAIN + 1, B_COUNT = B_TURN + 2
};
static_assert(B_COUNT * 8 + 16 <= 256, "barrier block");
static_assert(SMEM <= 232448, "shared memory per CTA");
}  // namespace pp

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st8u(uint32_t taddr, const uint32_t* v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// Named barrier over `count` threads that also returns the AND of `pred` over them.
__device__ __forceinline__ bool named_bar_and(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n.reg .pred p, q;\nsetp.ne.u32 p, %1, 0;\n"
        "barrier.cta.red.and.pred q, %2, %3, p;\nselp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// p = 2^(x * scale + neg_m) for the 128 scores of a row, written as bf16 pairs
// (round to nearest) over TMEM columns [0, 64) of the row's S buffer; returns
// the row sum of p in fp32.
__device__ __forceinline__ float exp_row_to_tmem(const float* x, float scale, float neg_m, uint32_t tP) {
    float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float e0 = ex2(fmaf(x[16 * c + 2 * k], scale, neg_m));
            const float e1 = ex2(fmaf(x[16 * c + 2 * k + 1], scale, neg_m));
            l4[(2 * k) & 3] += e0;
            l4[(2 * k + 1) & 3] += e1;
            pk[k] = pack_bf16(e0, e1);
        }
        tmem_st8u(tP + 8 * c, pk);
    }
    return (l4[0] + l4[1]) + (l4[2] + l4[3]);
}

__global__ void __launch_bounds__(pp::kThreads, 1)
    attention_pp_kernel(const __grid_constant__ LayerArgs a, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_o) {
    using namespace pp;
    extern __shared__ __align__(1024) uint8_t smem[];
    // 128B-swizzled tiles need a 1024-byte aligned base: report and leave if not
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicOr(a.flags, FLAG_INTERNAL);
        return;
    }
    // the delta update of this pass reads nothing this kernel writes: it may
    // start on SMs this grid leaves idle
    pdl_launch_dependents();
    const uint32_t sb = smem_u32(smem);
    uint64_t* bars = (uint64_t*)(smem + BAR);
    uint32_t* tmem_slot = (uint32_t*)(bars + B_COUNT);
    volatile int* abort_word = (volatile int*)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y, b = blockIdx.z;
    const int T = a.T;
    const int nq = (T + kTile - 1) / kTile;
    const int qtA = 2 * blockIdx.x;
    const bool hasB = qtA + 1 < nq;
    const int n = (a.T_kv + kTile - 1) / kTile;  // key blocks
    const bool inter = a.inter != 0;
    const int bh = b * a.H + h;
    const int xh = h * 128;
    // K stages that receive W_hi / W_lo at the end (free once the score products
    // of key blocks n-3 / n-2 have completed; stages no block uses when n is small)
    const int wst_hi = n >= 3 ? (n - 3) % kKStages : 2;
    const int wst_lo = n >= 2 ? (n - 2) % kKStages : 1;

    if (threadIdx.x == kLoadWarp * 32) {
        // the producer initialises the barriers and starts the first loads before
        // the block synchronises (the loads land on its own barriers)
        for (int i = 0; i < B_COUNT; ++i)
            mbar_init(&bars[i], (i == B_PFULL || i == B_PFULL + 1 || i == B_TURN || i == B_TURN + 1) ? 128 : 1);
        *abort_word = 0;
        fence_mbar_init();
        fence_async_smem();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        mbar_expect_tx(&bars[B_QA], kTileBytes);
        tma_load_3d(sb + QA, &tm_q, &bars[B_QA], xh, qtA * kTile, b);
        tma_load_3d(sb + QA + kHalf, &tm_q, &bars[B_QA], xh + 64, qtA * kTile, b);
        mbar_expect_tx(&bars[B_KFULL], kTileBytes);
        tma_load_3d(sb + K0, &tm_k, &bars[B_KFULL], xh, 0, b);
        tma_load_3d(sb + K0 + kHalf, &tm_k, &bars[B_KFULL], xh + 64, 0, b);
        if (hasB) {
            mbar_expect_tx(&bars[B_QB], kTileBytes);
            tma_load_3d(sb + QB, &tm_q, &bars[B_QB], xh, (qtA + 1) * kTile, b);
            tma_load_3d(sb + QB + kHalf, &tm_q, &bars[B_QB], xh + 64, (qtA + 1) * kTile, b);
        }
        for (int j = 1; j < kKStages && j < n; ++j) {
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

    if (warp == kLoadVWarp) {
        // ------------------------------------------------ TMA producer: V ring
        if (lane == 0) {
            tma_prefetch_desc(&tm_v);
            // (a fault test may switch this producer off: the MMA issuer's wait for V
            // then expires, and the kernel reports a timeout and unwinds)
            for (int j = 0; j < n && !a.dbg_skip_v; ++j) {
                const int vs = j % kVStages;
                if (j >= kVStages &&
                    !mbar_wait(&bars[B_VEMPTY + vs], ((j / kVStages) + 1) & 1, abort_word, a.flags, a.wait_ns))
                    break;
                mbar_expect_tx(&bars[B_VFULL + vs], kTileBytes);
                tma_load_3d(sb + V0 + vs * kTileBytes, &tm_v, &bars[B_VFULL + vs], xh, j * kTile, b);
                tma_load_3d(sb + V0 + vs * kTileBytes + kHalf, &tm_v, &bars[B_VFULL + vs], xh + 64, j * kTile, b);
            }
        }
        __syncwarp();
    } else if (warp == kLoadWarp) {
        // ------------------------------------------------ TMA producer: K ring, then W
        if (lane == 0) {
            tma_prefetch_desc(&tm_w);
            bool ok = true;
            for (int j = kKStages; j < n && ok; ++j) {
                const int ks = j % kKStages;
                if (!(ok = mbar_wait(&bars[B_KEMPTY + ks], ((j / kKStages) + 1) & 1, abort_word, a.flags, a.wait_ns))) break;
                mbar_expect_tx(&bars[B_KFULL + ks], kTileBytes);
                tma_load_3d(sb + K0 + ks * kTileBytes, &tm_k, &bars[B_KFULL + ks], xh, j * kTile, b);
                tma_load_3d(sb + K0 + ks * kTileBytes + kHalf, &tm_k, &bars[B_KFULL + ks], xh + 64, j * kTile, b);
            }
            if (inter && ok && n >= 3)
                ok = mbar_wait(&bars[B_KEMPTY + wst_hi], ((n - 3) / kKStages) & 1, abort_word, a.flags, a.wait_ns);
            if (inter && ok && n >= 2)
                ok = mbar_wait(&bars[B_KEMPTY + wst_lo], ((n - 2) / kKStages) & 1, abort_word, a.flags, a.wait_ns);
            // W comes from the prep kernel, which may still be running when this
            // grid starts (programmatic dependent launch): wait for it here
            if (inter) pdl_wait_primary();
            if (inter && ok) {
                const int nbh = a.B * a.H;
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
        if (lane == 0) {
            constexpr uint32_t ID_KK = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t ID_KMN = idesc_bf16(128, 128, 0, 1);
            const int ntile = hasB ? 2 : 1;
            // S_t(0) = Q_t K_0^T
            if (!(mbar_wait(&bars[B_KFULL], 0, abort_word, a.flags, a.wait_ns))) goto drain;
            for (int t = 0; t < ntile; ++t) {
                if (!(mbar_wait(&bars[B_QA + t], 0, abort_word, a.flags, a.wait_ns))) goto drain;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + t * 128, kmajor_desc(sb + QA + t * kTileBytes, kk), kmajor_desc(sb + K0, kk),
                             ID_KK, kk > 0);
                mma_commit(&bars[B_SFULL + t]);
            }
            mma_commit(&bars[B_KEMPTY]);
            for (int j = 0; j < n; ++j) {
                const int vs = j % kVStages;
                const int ks1 = (j + 1) % kKStages;
                for (int t = 0; t < ntile; ++t) {
                    // O_t += P_t(j) V_j (P_t in TMEM over the first columns of S_t)
                    if (!(mbar_wait(&bars[B_PFULL + t], j & 1, abort_word, a.flags, a.wait_ns))) goto drain;
                    if (t == 0 && !(mbar_wait(&bars[B_VFULL + vs], (j / kVStages) & 1, abort_word, a.flags, a.wait_ns)))
                        goto drain;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8,
                                    mnmajor_desc(sb + V0 + vs * kTileBytes, kk), ID_KMN, (j > 0 || kk > 0));
                    mma_commit(&bars[B_PVDONE + t]);
                    if (t == ntile - 1) mma_commit(&bars[B_VEMPTY + vs]);
                    if (j + 1 < n) {
                        // S_t(j+1) = Q_t K_{j+1}^T into S_t, once P_t(j) has been read
                        if (t == 0 &&
                            !(mbar_wait(&bars[B_KFULL + ks1], ((j + 1) / kKStages) & 1, abort_word, a.flags, a.wait_ns)))
                            goto drain;
                        if (!(mbar_wait(&bars[B_PVDONE + t], j & 1, abort_word, a.flags, a.wait_ns))) goto drain;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_bf16(tmem + t * 128, kmajor_desc(sb + QA + t * kTileBytes, kk),
                                     kmajor_desc(sb + K0 + ks1 * kTileBytes, kk), ID_KK, kk > 0);
                        mma_commit(&bars[B_SFULL + t]);
                        if (t == ntile - 1) mma_commit(&bars[B_KEMPTY + ks1]);
                    }
                }
            }
            // O_inter_t = Q_t W_hi + Q_t W_lo into S_t (free once P_t(n-1) V has completed)
            if (inter && !(mbar_wait(&bars[B_W], 0, abort_word, a.flags, a.wait_ns))) goto drain;
            for (int t = 0; t < ntile; ++t) {
                if (inter) {
                    if (!(mbar_wait(&bars[B_PVDONE + t], (n - 1) & 1, abort_word, a.flags, a.wait_ns))) goto drain;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tmem + t * 128, kmajor_desc(sb + QA + t * kTileBytes, kk),
                                 mnmajor_desc(sb + K0 + wst_hi * kTileBytes, kk), ID_KMN, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tmem + t * 128, kmajor_desc(sb + QA + t * kTileBytes, kk),
                                 mnmajor_desc(sb + K0 + wst_lo * kTileBytes, kk), ID_KMN, 1);
                }
                mma_commit(&bars[B_OIDONE + t]);
            }
        drain:
            // (a failed wait has already set the abort word and the TIMEOUT flag)
            // every MMA issued so far completes before TMEM is released
            mma_commit(&bars[B_DRAIN]);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&bars[B_DRAIN]), 0) && globaltimer_ns() - t0 < a.wait_ns) {
            }
        }
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------ softmax + epilogue of tile t
        const int t = warp >> 2;
        if (t == 0 || hasB) {
            const int r = (warp & 3) * 32 + lane;
            const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
            const uint32_t tS = tmem + t * 128 + lrow;
            const uint32_t tO = tmem + 256 + t * 128 + lrow;
            const float scale = a.sm_scale_log2;
            float m = 0.f, l = 0.f;
            float x[128];
            bool ok = true;
            for (int j = 0; j < n; ++j) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL + t], j & 1, abort_word, a.flags, a.wait_ns));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, x + 32 * c);
                tmem_ld_wait();
                const int valid = a.T_kv - j * kTile;
                if (valid < 128) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c >= valid) x[c] = -INFINITY;
                }
                if (j == 0) m = row_max<128>(x) * scale;  // the first block's row max sets the offset
                // the two tiles take turns on the MUFU pipe: tile B's exponentials of
                // block j start after tile A's, tile A's of block j+1 after tile B's
                // of block j, so each tile's products run while the other one exponentiates
                if (hasB && (t == 1 || j > 0)) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_TURN + t], (t == 1 ? j : j - 1) & 1, abort_word,
                                                           a.flags, a.wait_ns));
                    if (!ok) break;
                }
                float lt = exp_row_to_tmem(x, scale, -m, tS);
                const bool redo = !(lt < 9.2233720e18f);  // >= 2^63, inf or NaN
                if (__any_sync(0xffffffffu, redo)) {
                    // the offset is too low for this block (or a score is not finite):
                    // move it to the row's max, rescale O and l, redo P_t(j)
                    float f = 1.0f;
                    if (redo) {
                        const float mn = fmaxf(m, row_max<128>(x) * scale);
                        f = ex2(m - mn);
                        m = mn;
                    }
                    if (j > 0) {
                        // (in 8-column pieces: the 128 scores stay live in registers)
#pragma unroll 1
                        for (int c = 0; c < 128; c += 8) {
                            float o[8];
                            uint32_t ou[8];
                            tmem_ld8(tO + c, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int q = 0; q < 8; ++q) ou[q] = __float_as_uint(o[q] * f);
                            tmem_st8u(tO + c, ou);
                        }
                    }
                    l *= f;
                    lt = exp_row_to_tmem(x, scale, -m, tS);
                }
                l += lt;
                if (hasB && (t == 0 || j + 1 < n)) mbar_arrive(&bars[B_TURN + (t ^ 1)]);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars[B_PFULL + t]);
            }
            // epilogue: out = a O / l + O_inter, one bf16 rounding, through the Q buffer
            const bool e_ok =
                __all_sync(0xffffffffu, ok && mbar_wait(&bars[B_OIDONE + t], 0, abort_word, a.flags, a.wait_ns));
            const int q0 = (qtA + t) * kTile;
            const int tok = q0 + r;
            if (e_ok) {
                tc_fence_after();
                const float inv_l = 1.0f / l;
                const float inv_out = a.mix ? inv_l * a.mix[bh * 2] : inv_l;
                const uint32_t qbuf = (t == 0 ? QA : QB);
#pragma unroll 1
                for (int c = 0; c < 128; c += 32) {
                    float o[32], e[32];
                    tmem_ld32(tO + c, o);
                    if (inter) tmem_ld32(tS + c, e);
                    tmem_ld_wait();
                    if (!inter) {
                        if (a.oi_ext && tok < T) {
                            // token-level access: the read comes from the token-level kernels
                            const float4* src = reinterpret_cast<const float4*>(
                                a.oi_ext + (((size_t)b * T + tok) * a.H + h) * 128 + c);
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
                    }
                    if (a.out) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 w;
                            w.x = pack_bf16(fmaf(o[8 * q + 0], inv_out, e[8 * q + 0]), fmaf(o[8 * q + 1], inv_out, e[8 * q + 1]));
                            w.y = pack_bf16(fmaf(o[8 * q + 2], inv_out, e[8 * q + 2]), fmaf(o[8 * q + 3], inv_out, e[8 * q + 3]));
                            w.z = pack_bf16(fmaf(o[8 * q + 4], inv_out, e[8 * q + 4]), fmaf(o[8 * q + 5], inv_out, e[8 * q + 5]));
                            w.w = pack_bf16(fmaf(o[8 * q + 6], inv_out, e[8 * q + 6]), fmaf(o[8 * q + 7], inv_out, e[8 * q + 7]));
                            // column chunk (c + 8q) / 8 of the row, in box c / 64
                            const int chunk = (c % 64) / 8 + q;
                            *reinterpret_cast<uint4*>(smem + qbuf + (c / 64) * kHalf + sw128_offset(r, chunk)) = w;
                        }
                    }
                    if (a.out_intra && tok < T) {
                        const size_t row = (((size_t)b * T + tok) * a.H + h) * 128 + c;
                        float4* di = reinterpret_cast<float4*>(a.out_intra + row);
                        float4* de = reinterpret_cast<float4*>(a.out_inter + row);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            di[q] = make_float4(o[4 * q] * inv_l, o[4 * q + 1] * inv_l, o[4 * q + 2] * inv_l,
                                                o[4 * q + 3] * inv_l);
                            de[q] = make_float4(e[4 * q], e[4 * q + 1], e[4 * q + 2], e[4 * q + 3]);
                        }
                    }
                }
                if (a.out) fence_async_smem();
            }
            // the four warps of the tile meet here (no early exit); the tile is
            // stored only if all of them wrote their rows
            const bool all_ok = named_bar_and(1 + t, 128, e_ok);
            if (a.out && all_ok && (threadIdx.x & 127) == 0) {
                const uint32_t qbuf = (t == 0 ? QA : QB);
                // rows past T are clipped by the tensor map
                tma_store_3d(&tm_o, sb + qbuf, xh, q0, b);
                tma_store_3d(&tm_o, sb + qbuf + kHalf, xh + 64, q0, b);
                bulk_commit_group();
                bulk_wait_read_all();
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
