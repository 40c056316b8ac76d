// tc_kernels.cuh -- tensor-core (tcgen05 / TMEM / TMA) kernels of the hybrid
// layer for bf16 I/O and d = 128 on sm_100a.
//
// Source: "Technical summary: Attend Locally, Remember Linearly (ARL2)",
// gist.science/ar/paper/2605.16579, §2.1 (intra-frame softmax branch,
// inter-frame read O_inter = Q' S_{N-1}, gated delta update) and §2.2
// (frame-level access: all tokens read the pre-update state).
//
// intra_frame_attention: one CTA per (128-query tile, head, batch).  Warp 4
// streams Q, K and V tiles with TMA into 128B-swizzled shared memory; warp 5
// issues the tcgen05 MMAs; warps 0-3 own one query row per thread and run the
// online softmax from TMEM.  Before the key loop the same Q tile is multiplied
// by W = phi_q^T S_{N-1} (passed as a two-term bf16 split W_hi + W_lo), so the
// inter-frame read lands in TMEM next to the softmax accumulator and the
// epilogue writes out = O_intra + O_inter once.
//   TMEM columns: [0,128) S buffer 0, [128,256) S buffer 1, [256,384) O,
//                 [384,512) O_inter.
//   Shared memory: Q 32 KB | K 2 x 32 KB | V 2 x 32 KB | P 2 x 32 KB (the P
//                 buffers hold W_hi / W_lo until the first softmax).
//
// delta_update_partials: one CTA per (token split, head, batch).  Per 128-token
// tile: K~ = K phi_k^T on the tensor core, row L2-normalisation and beta in
// registers, then G += (beta K')^T K' and P += (beta K')^T V as MN-major
// contractions over the tokens, with beta K' and K' split into bf16 hi + lo
// (G takes hi*hi + hi*lo + lo*hi, P takes hi*V + lo*V; V is exact in bf16).
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace hyb {
namespace tc {

using namespace sm100;

constexpr int kTile = 128;
constexpr uint32_t kTileBytes = 128 * 128 * 2;  // one 128 x 128 bf16 tile
constexpr uint32_t kHalf = kTileBytes / 2;      // one 128 x 64 TMA box

// ============================================================== attention
namespace attn {
constexpr uint32_t Q = 0;
constexpr uint32_t K0 = Q + kTileBytes;
constexpr uint32_t V0 = K0 + 2 * kTileBytes;
constexpr uint32_t P0 = V0 + 2 * kTileBytes;
constexpr uint32_t BAR = P0 + 2 * kTileBytes;
constexpr uint32_t SMEM = 1024 + BAR + 256;  // + alignment slack + barriers
constexpr int kThreads = 192;
enum { B_Q = 0, B_KFULL = 1, B_KEMPTY = 3, B_VFULL = 5, B_VEMPTY = 7, B_SFULL = 9, B_PFULL = 11,
       B_PVDONE = 13, B_COUNT = 15 };
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

__global__ void __launch_bounds__(attn::kThreads, 1)
    attention_kernel(const __grid_constant__ LayerArgs a, const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_w) {
    using namespace attn;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    uint64_t* bars = (uint64_t*)(smem + BAR);
    uint32_t* tmem_slot = (uint32_t*)(bars + B_COUNT);
    volatile int* abort_word = (volatile int*)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int T = a.T;
    const int q0 = qt * kTile;
    const int n = (T + kTile - 1) / kTile;
    const int bh = b * a.H + h;

    if (threadIdx.x == 0) {
        for (int i = 0; i < B_COUNT; ++i) mbar_init(&bars[i], i == B_PFULL || i == B_PFULL + 1 ? 128 : 1);
        *abort_word = 0;
        fence_mbar_init();
    }
    if (warp == 5) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS0 = tmem, tO = tmem + 256, tOI = tmem + 384;

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_w);
            const int xh = h * 128;
            mbar_expect_tx(&bars[B_Q], 3 * kTileBytes);
            tma_load_3d(sb + Q, &tm_q, &bars[B_Q], xh, q0, b);
            tma_load_3d(sb + Q + kHalf, &tm_q, &bars[B_Q], xh + 64, q0, b);
            const int nbh = a.B * a.H;
            tma_load_3d(sb + P0, &tm_w, &bars[B_Q], 0, 0, bh);
            tma_load_3d(sb + P0 + kHalf, &tm_w, &bars[B_Q], 64, 0, bh);
            tma_load_3d(sb + P0 + kTileBytes, &tm_w, &bars[B_Q], 0, 0, nbh + bh);
            tma_load_3d(sb + P0 + kTileBytes + kHalf, &tm_w, &bars[B_Q], 64, 0, nbh + bh);
            for (int j = 0; j < n; ++j) {
                const int s = j & 1;
                const uint32_t par = ((j >> 1) + 1) & 1;
                if (j >= 2 && !mbar_wait(&bars[B_KEMPTY + s], par, abort_word, a.flags)) break;
                mbar_expect_tx(&bars[B_KFULL + s], kTileBytes);
                tma_load_3d(sb + K0 + s * kTileBytes, &tm_k, &bars[B_KFULL + s], xh, j * kTile, b);
                tma_load_3d(sb + K0 + s * kTileBytes + kHalf, &tm_k, &bars[B_KFULL + s], xh + 64, j * kTile, b);
                if (j >= 2 && !mbar_wait(&bars[B_VEMPTY + s], par, abort_word, a.flags)) break;
                mbar_expect_tx(&bars[B_VFULL + s], kTileBytes);
                tma_load_3d(sb + V0 + s * kTileBytes, &tm_v, &bars[B_VFULL + s], xh, j * kTile, b);
                tma_load_3d(sb + V0 + s * kTileBytes + kHalf, &tm_v, &bars[B_VFULL + s], xh + 64, j * kTile, b);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_KK = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t ID_KMN = idesc_bf16(128, 128, 0, 1);
            bool ok = mbar_wait(&bars[B_Q], 0, abort_word, a.flags);
            if (ok) {
                tc_fence_after();
                // O_inter = Q W_hi + Q W_lo
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tOI, kmajor_desc(sb + Q, kk), kmajor_desc(sb + P0, kk), ID_KK, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tOI, kmajor_desc(sb + Q, kk), kmajor_desc(sb + P0 + kTileBytes, kk), ID_KK, 1);
                for (int j = 0; j < 2 && j < n && ok; ++j) {
                    ok = mbar_wait(&bars[B_KFULL + j], 0, abort_word, a.flags);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tS0 + j * 128, kmajor_desc(sb + Q, kk),
                                 kmajor_desc(sb + K0 + j * kTileBytes, kk), ID_KK, kk > 0);
                    mma_commit(&bars[B_SFULL + j]);
                    mma_commit(&bars[B_KEMPTY + j]);
                }
            }
            for (int j = 0; j < n && ok; ++j) {
                const int s = j & 1;
                const uint32_t par = (j >> 1) & 1;
                if (!mbar_wait(&bars[B_PFULL + s], par, abort_word, a.flags)) break;
                if (!mbar_wait(&bars[B_VFULL + s], par, abort_word, a.flags)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tO, kmajor_desc(sb + P0 + s * kTileBytes, kk),
                             mnmajor_desc(sb + V0 + s * kTileBytes, kk), ID_KMN, (j > 0 || kk > 0));
                mma_commit(&bars[B_PVDONE + s]);
                mma_commit(&bars[B_VEMPTY + s]);
                if (j + 2 < n) {
                    if (!mbar_wait(&bars[B_KFULL + s], ((j + 2) >> 1) & 1, abort_word, a.flags)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tS0 + s * 128, kmajor_desc(sb + Q, kk),
                                 kmajor_desc(sb + K0 + s * kTileBytes, kk), ID_KK, kk > 0);
                    mma_commit(&bars[B_SFULL + s]);
                    mma_commit(&bars[B_KEMPTY + s]);
                }
            }
            // drain: every MMA issued so far completes before TMEM is released
            mma_commit(&bars[B_Q]);
            uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&bars[B_Q]), 1) && globaltimer_ns() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax + epilogue (row r)
        const int r = threadIdx.x;  // 0..127, TMEM lane r
        const uint32_t lrow = (uint32_t)(warp * 32) << 16;
        const float scale = a.sm_scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        float x[128];
        for (int j = 0; j < n; ++j) {
            const int s = j & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL + s], (j >> 1) & 1, abort_word, a.flags));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS0 + s * 128 + lrow + c * 32, x + c * 32);
            tmem_ld_wait();
            const int valid = T - j * kTile;
            if (valid < kTile) {
#pragma unroll
                for (int i = 0; i < 128; ++i)
                    if (i >= valid) x[i] = -INFINITY;
            }
            // row max of the raw scores: eight independent chains, then a tree
            float m8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = x[k];
#pragma unroll
            for (int i = 8; i < 128; i += 8)
#pragma unroll
                for (int k = 0; k < 8; ++k) m8[k] = fmaxf(m8[k], x[i + k]);
            const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * scale;
            if (j == 0) {
                m = mx;
            } else if (mx > m + 8.0f) {
                // the running max moved by more than 2^8: rescale O (after PV_{j-1})
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PVDONE + ((j - 1) & 1)], ((j - 1) >> 1) & 1,
                                                         abort_word, a.flags));
                if (!ok) break;
                tc_fence_after();
                const float f = ex2(m - mx);
                l *= f;
                float o[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    tmem_ld32(tO + lrow + c * 32, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= f;
                    tmem_st32(tO + lrow + c * 32, o);
                }
                tmem_st_wait();
                m = mx;
            }
            const float neg_m = -m;
            if (j >= 2) {
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&bars[B_PVDONE + s], ((j >> 1) + 1) & 1, abort_word, a.flags));
                if (!ok) break;
            }
            uint8_t* P = smem + P0 + s * kTileBytes;
            float sum8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) sum8[k] = 0.f;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float* v = x + hf * 64 + c * 8;
                    float e[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        e[k] = ex2(fmaf(v[k], scale, neg_m));
                        sum8[k] += e[k];
                    }
                    uint4 w;
                    w.x = pack_bf16(e[0], e[1]);
                    w.y = pack_bf16(e[2], e[3]);
                    w.z = pack_bf16(e[4], e[5]);
                    w.w = pack_bf16(e[6], e[7]);
                    *reinterpret_cast<uint4*>(P + hf * kHalf + sw128_offset(r, c)) = w;
                }
            l += ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_PFULL + s]);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PVDONE + ((n - 1) & 1)], ((n - 1) >> 1) & 1,
                                                        abort_word, a.flags));
        if (ok) {
            tc_fence_after();
            const int t = q0 + r;
            const float inv_l = 1.0f / l;
            const size_t row = (((size_t)b * T + t) * a.H + h) * 128;
            float o[32], e[32];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                tmem_ld32(tO + lrow + c * 32, o);
                tmem_ld32(tOI + lrow + c * 32, e);
                tmem_ld_wait();
                if (t < T) {
                    if (a.out) {
                        uint4* dst = reinterpret_cast<uint4*>((__nv_bfloat16*)a.out + row + c * 32);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 w;
                            w.x = pack_bf16(o[8 * q + 0] * inv_l + e[8 * q + 0], o[8 * q + 1] * inv_l + e[8 * q + 1]);
                            w.y = pack_bf16(o[8 * q + 2] * inv_l + e[8 * q + 2], o[8 * q + 3] * inv_l + e[8 * q + 3]);
                            w.z = pack_bf16(o[8 * q + 4] * inv_l + e[8 * q + 4], o[8 * q + 5] * inv_l + e[8 * q + 5]);
                            w.w = pack_bf16(o[8 * q + 6] * inv_l + e[8 * q + 6], o[8 * q + 7] * inv_l + e[8 * q + 7]);
                            dst[q] = w;
                        }
                    }
                    if (a.out_intra) {
                        float4* di = reinterpret_cast<float4*>(a.out_intra + row + c * 32);
                        float4* de = reinterpret_cast<float4*>(a.out_inter + row + c * 32);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            di[q] = make_float4(o[4 * q] * inv_l, o[4 * q + 1] * inv_l, o[4 * q + 2] * inv_l,
                                                o[4 * q + 3] * inv_l);
                            de[q] = make_float4(e[4 * q], e[4 * q + 1], e[4 * q + 2], e[4 * q + 3]);
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 512);
}

// ============================================================== update partials
namespace upd {
constexpr uint32_t PHI = 0;
constexpr uint32_t KT = PHI + kTileBytes;
constexpr uint32_t VT = KT + kTileBytes;
constexpr uint32_t AH = VT + kTileBytes;
constexpr uint32_t AL = AH + kTileBytes;
constexpr uint32_t KH = AL + kTileBytes;
constexpr uint32_t KL = KH + kTileBytes;
constexpr uint32_t BAR = KL + kTileBytes;
constexpr uint32_t SMEM = 1024 + BAR + 256;
constexpr int kThreads = 192;
enum { B_PHI = 0, B_KFULL, B_KFREE, B_VFULL, B_KTFULL, B_OPSFULL, B_OPSFREE, B_COUNT };
}  // namespace upd

__global__ void __launch_bounds__(upd::kThreads, 1)
    partials_kernel(const __grid_constant__ LayerArgs a, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_phik) {
    using namespace upd;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    uint64_t* bars = (uint64_t*)(smem + BAR);
    uint32_t* tmem_slot = (uint32_t*)(bars + B_COUNT);
    volatile int* abort_word = (volatile int*)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int T = a.T;
    const int bh = b * a.H + h;
    const int t_begin = split * a.split_tokens;
    const int t_end = min(T, t_begin + a.split_tokens);
    const int nt = (t_end - t_begin + kTile - 1) / kTile;

    if (threadIdx.x == 0) {
        for (int i = 0; i < B_COUNT; ++i) mbar_init(&bars[i], i == B_OPSFULL ? 128 : 1);
        *abort_word = 0;
        fence_mbar_init();
    }
    if (warp == 5) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tKT = tmem, tG = tmem + 128, tP = tmem + 256;

    if (warp == 4) {
        if (lane == 0) {
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
    } else if (warp == 5) {
        if (lane == 0) {
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
                    const uint32_t first = (i > 0 || kk > 0);
                    mma_bf16(tG, mnmajor_desc(sb + AH, kk), mnmajor_desc(sb + KH, kk), ID_MNMN, first);
                    mma_bf16(tG, mnmajor_desc(sb + AH, kk), mnmajor_desc(sb + KL, kk), ID_MNMN, 1);
                    mma_bf16(tG, mnmajor_desc(sb + AL, kk), mnmajor_desc(sb + KH, kk), ID_MNMN, 1);
                    mma_bf16(tP, mnmajor_desc(sb + AH, kk), mnmajor_desc(sb + VT, kk), ID_MNMN, first);
                    mma_bf16(tP, mnmajor_desc(sb + AL, kk), mnmajor_desc(sb + VT, kk), ID_MNMN, 1);
                }
                mma_commit(&bars[B_OPSFREE]);
            }
            mma_commit(&bars[B_PHI]);
            uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&bars[B_PHI]), 1) && globaltimer_ns() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
    } else {
        const int r = threadIdx.x;  // token row within the tile, TMEM lane r
        const uint32_t lrow = (uint32_t)(warp * 32) << 16;
        bool ok = true;
        float x[128];
        for (int i = 0; i < nt; ++i) {
            const uint32_t par = i & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_KTFULL], par, abort_word, a.flags));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tKT + lrow + c * 32, x + c * 32);
            tmem_ld_wait();
            const int tok = t_begin + i * kTile + r;
            const bool valid = tok < t_end;
            float ss = 0.f;
#pragma unroll
            for (int c = 0; c < 128; ++c) ss = fmaf(x[c], x[c], ss);
            const float inv = valid ? 1.0f / sqrtf(ss + a.l2_eps) : 0.f;
            const float beta = valid ? sigmoidf_(a.beta_logits[(size_t)bh * T + tok]) : 0.f;
            if (i > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_OPSFREE], (i - 1) & 1, abort_word, a.flags));
                if (!ok) break;
            }
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t ah[4], al[4], kh[4], kl[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int col = hf * 64 + c * 8 + 2 * q;
                        float k0 = x[col] * inv, k1 = x[col + 1] * inv;
                        float a0 = k0 * beta, a1 = k1 * beta;
                        __nv_bfloat162 khv = __floats2bfloat162_rn(k0, k1);
                        __nv_bfloat162 ahv = __floats2bfloat162_rn(a0, a1);
                        kh[q] = *reinterpret_cast<uint32_t*>(&khv);
                        ah[q] = *reinterpret_cast<uint32_t*>(&ahv);
                        kl[q] = pack_bf16(k0 - __low2float(khv), k1 - __high2float(khv));
                        al[q] = pack_bf16(a0 - __low2float(ahv), a1 - __high2float(ahv));
                    }
                    const uint32_t off = hf * kHalf + sw128_offset(r, c);
                    *reinterpret_cast<uint4*>(smem + AH + off) = make_uint4(ah[0], ah[1], ah[2], ah[3]);
                    *reinterpret_cast<uint4*>(smem + AL + off) = make_uint4(al[0], al[1], al[2], al[3]);
                    *reinterpret_cast<uint4*>(smem + KH + off) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
                    *reinterpret_cast<uint4*>(smem + KL + off) = make_uint4(kl[0], kl[1], kl[2], kl[3]);
                }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_OPSFULL]);
        }
        if (ok && nt > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_OPSFREE], (nt - 1) & 1, abort_word, a.flags));
        if (ok) {
            tc_fence_after();
            // row r of G and P (TMEM lane = output row i)
            float* dst = a.partials + (((size_t)bh * a.nsplit + split) * 128 + r) * 256;
            float v[32];
            for (int c = 0; c < 4; ++c) {
                if (nt > 0) {
                    tmem_ld32(tG + lrow + c * 32, v);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) v[q] = 0.f;
                }
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    reinterpret_cast<float4*>(dst + c * 32)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
            for (int c = 0; c < 4; ++c) {
                if (nt > 0) {
                    tmem_ld32(tP + lrow + c * 32, v);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) v[q] = 0.f;
                }
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    reinterpret_cast<float4*>(dst + 128 + c * 32)[q] =
                        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 512);
}

}  // namespace tc
}  // namespace hyb
